// Chunked prefill over the quantized paged cache (sm_100a, tcgen05 tensor cores).
//
// A chunk of q_len new tokens (already quantised into the cache by
// kvq_append) attends causally to the cache and to itself: row r of the chunk,
// at absolute position len - q_len + r, sees positions 0 .. len - q_len + r
// (keep the cache, process only the new tokens: "Reutilizacao de Cache KV para
// Conversas Longas no Apple Silicon", "Principais Descobertas e Benchmarks";
// exact softmax attention through the flash-attention path: KVSplit page,
// "Exemplos de uso e opcoes de CLI").
//
// Two passes:
//  1. dequant_tiles_kernel: every (sequence, KV head) of the batch is
//     dequantised once, in 64-token tiles of a workspace: K as two fp16 tiles
//     K_hi = fp16(k^) and K_lo = fp16(k^ - K_hi) [64 tokens][D] (fp16 alone
//     would round the x10 outlier key channels by up to 2^-12 relative, which
//     moves the softmax by ~0.2%; hi + lo keeps ~22 bits), and V transposed
//     [D][64 tokens] in fp16, so both MMAs read K-major operands.
//     (Dequantising inside the attention kernel would redo it for every
//     128-row query tile: a 4096-token chunk with 4 query heads per KV head
//     has 128 of them.)  Positions past the end are zero.
//  2. prefill_attn_kernel: one CTA per (query tile of 128 rows = 128/G tokens
//     x G query heads of one KV head).  Warp 0 streams Q once and the K_hi /
//     K_lo / V tiles through a three-stage ring with 2-D / 3-D TMA tensor
//     loads (128-byte swizzle); warp 1 owns TMEM (S double buffer + O
//     accumulator) and issues tcgen05.mma kind::f16 (fp16 x fp16 -> fp32):
//        S_j = Q K_hi,j^T + Q K_lo,j^T into TMEM, O += P_j V_j from shared memory;
//     warps 2-5 (one per TMEM lane quadrant, one thread per row) read S with
//     tcgen05.ld, apply sigma log2 e and the causal mask, run the online softmax
//     (running max moved only when it grows by more than 2^8; then O is
//     rescaled in TMEM), write P as fp16 in the swizzled K-major layout, and at
//     the end normalise O and store it.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "kvq_internal.cuh"
#include "sm100_util.cuh"
#include "tcgen05_util.cuh"
#include "tma_host.h"

namespace kvq {
namespace {

constexpr int kQT = 128;     // rows per query tile (MMA M)
constexpr int kKT = 64;      // tokens per K / V tile (MMA N of S, K of P V)

struct PrefillSeq {
  int32_t seq_id;
  int32_t len;        // tokens in the cache, chunk included
  int32_t q_len;      // chunk rows
  int32_t q_off;      // first row of this sequence in q / out
  int32_t tile_base;  // first workspace tile of this sequence (KV head 0)
  int32_t n_tiles;    // tiles per KV head = ceil(len / 64)
  int32_t qt_begin;   // first query tile of this sequence in the grid
  int32_t pad;
};

struct PrefillBatch {
  int32_t n;
  int32_t H, G, Hq;
  PrefillSeq s[kMaxBatch];
};

__device__ __forceinline__ int find_seq_by(const PrefillBatch& b, int x, bool by_tiles) {
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int key = by_tiles ? b.s[mid].tile_base : b.s[mid].qt_begin;
    if (key <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ pass 1: dequantise
template <int D>
__global__ void __launch_bounds__(256) dequant_tiles_kernel(const Layout L, int layer,
                                                            const __grid_constant__ PrefillBatch b,
                                                            __half* __restrict__ khi, __half* __restrict__ klo,
                                                            __half* __restrict__ vws) {
  __shared__ __align__(16) __half vt[kKT][D + 8];
  const int gt = blockIdx.x;
  const int si = find_seq_by(b, gt, true);
  const PrefillSeq sq = b.s[si];
  const int rel = gt - sq.tile_base;
  const int h = rel / sq.n_tiles, j = rel % sq.n_tiles;
  const int tid = threadIdx.x;
  constexpr int NB = D / 32;
  constexpr int TPT = 256 / kKT;                 // threads per token
  constexpr int EPT = D / TPT;                   // elements per thread
  const int64_t tile_off = int64_t(gt) * kKT * D;

  const int t = tid / TPT, part = tid % TPT;
  const int pos = j * kKT + t;
  const uint8_t* blk = nullptr;
  int r = 0;
  if (pos < sq.len) {
    const int page = L.page_table[int64_t(sq.seq_id) * L.max_pages_per_seq + pos / L.page_tokens];
    if (page < 0 || page >= L.n_pages) {
      record_error(L.err, kErrBadPage);
    } else {
      blk = L.head_ptr(layer, page, h);
      r = pos % L.page_tokens;
    }
  }
  // 8 consecutive elements e0 .. e0+7 of this token's row, exact dequantised values in fp32
  auto deq = [&](int bits, const uint8_t* codes, const uint8_t* scales, int e0, float (&o)[8]) {
    if (!blk) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = 0.f;
      return;
    }
    if (bits == 16) {
      const uint4 w = *reinterpret_cast<const uint4*>(codes + int64_t(r) * D * 2 + e0 * 2);
      const __half* hv = reinterpret_cast<const __half*>(&w);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __half2float(hv[i]);
      return;
    }
    const float d = __half2float(reinterpret_cast<const __half*>(scales + int64_t(r) * NB * 2)[e0 / 32]);
    if (bits == 8) {
      const uint2 w = *reinterpret_cast<const uint2*>(codes + int64_t(r) * D + e0);
      const int8_t* c = reinterpret_cast<const int8_t*>(&w);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = d * float(c[i]);      // exact: 11 x 7 significant bits
    } else {
      const int blkoff = (e0 / 32) * 16, q = (e0 % 32) / 8;   // q = which 8-element quarter of the block
      const uint2 w = *reinterpret_cast<const uint2*>(codes + int64_t(r) * (D / 2) + blkoff + 8 * (q & 1));
      const uint8_t* by = reinterpret_cast<const uint8_t*>(&w);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = d * float((q < 2 ? (by[i] & 0xF) : (by[i] >> 4)) - 8);
    }
  };
#pragma unroll 1
  for (int g = 0; g < EPT / 8; ++g) {
    const int e0 = part * EPT + 8 * g;
    float x[8];
    __half hi[8], lo[8];
    deq(L.k_bits, blk, blk + L.k_scales_off, e0, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      hi[i] = __float2half_rn(x[i]);
      lo[i] = __float2half_rn(x[i] - __half2float(hi[i]));
    }
    *reinterpret_cast<uint4*>(khi + tile_off + t * D + e0) = *reinterpret_cast<uint4*>(hi);
    *reinterpret_cast<uint4*>(klo + tile_off + t * D + e0) = *reinterpret_cast<uint4*>(lo);
    deq(L.v_bits, blk + L.v_codes_off, blk + L.v_scales_off, e0, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) hi[i] = __float2half_rn(x[i]);
    *reinterpret_cast<uint4*>(&vt[t][e0]) = *reinterpret_cast<uint4*>(hi);
  }
  __syncthreads();
  // transposed V: vws tile [d][token]
  for (int item = tid; item < D * (kKT / 8); item += 256) {
    const int d = item / (kKT / 8), tg = item % (kKT / 8);
    __half o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = vt[8 * tg + i][d];
    *reinterpret_cast<uint4*>(vws + tile_off + d * kKT + 8 * tg) = *reinterpret_cast<uint4*>(o);
  }
}

// ------------------------------------------------------------------ pass 2: attention
template <int D>
struct PTraits {
  static constexpr int CB = D / 64;                      // 128-byte column blocks of a Q / K row
  static constexpr int NSTAGE = 3;
  static constexpr int Q_BYTES = kQT * D * 2;            // CB blocks of [128 rows][128 B]
  static constexpr int K_BYTES = kKT * D * 2;            // CB blocks of [64 rows][128 B]
  static constexpr int V_BYTES = D * kKT * 2;            // one block of [D rows][128 B]
  static constexpr int STAGE = 2 * K_BYTES + V_BYTES;    // K_hi, K_lo, V^T
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_P = OFF_KV + NSTAGE * STAGE;
  static constexpr int P_BYTES = kQT * kKT * 2;          // one block of [128 rows][128 B]
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  // + alignment slack; never less than ~116 KB so that a second CTA cannot
  // share the SM and wait in tcgen05.alloc
  static constexpr int SMEM_NEED = OFF_BAR + 256 + 1024;
  static constexpr int SMEM = SMEM_NEED > 118 * 1024 ? SMEM_NEED : 118 * 1024;
  static constexpr int NT = 192;                         // 6 warps
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL0 = 0, O_COL = 128;     // S double buffer [0, 128), O [128, 128 + D)
  static_assert(O_COL + D <= TMEM_COLS, "TMEM");
  static_assert(OFF_KV % 1024 == 0 && STAGE % 1024 == 0 && OFF_P % 1024 == 0, "swizzle atoms");
};

// barriers: 0 q_full | 1..3 kv_full | 4..6 kv_empty | 7..8 s_full | 9 p_full | 10 pv_done | 11 mma_done
struct PrefillArgs {
  float scale_log2;
  __half* out;
  uint32_t* err;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_khi,
                        const __grid_constant__ CUtensorMap tm_klo, const __grid_constant__ CUtensorMap tm_v,
                        const PrefillArgs a, const __grid_constant__ PrefillBatch b) {
  using T = PTraits<D>;
  constexpr int NS = T::NSTAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * i; };
  constexpr int B_Q = 0, B_FULL = 1, B_EMPTY = 1 + NS, B_S = 1 + 2 * NS, B_P = 3 + 2 * NS, B_PV = 4 + 2 * NS,
                B_DONE = 5 + 2 * NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int si = find_seq_by(b, blockIdx.x, false);
  const PrefillSeq sq = b.s[si];
  const int G = b.G, TT = kQT / G;                        // tokens per query tile
  const int nq = (sq.q_len + TT - 1) / TT;
  const int qt = nq - 1 - (int(blockIdx.x) - sq.qt_begin); // heavy tiles first
  const int h = blockIdx.y;
  const int tok0 = qt * TT;                                // first chunk row of this tile
  const int qpos0 = sq.len - sq.q_len + tok0;              // absolute position of row 0
  const int qpos_last = sq.len - sq.q_len + min(tok0 + TT, sq.q_len) - 1;
  const int n_kv = qpos_last / kKT + 1;
  const int tile_base = sq.tile_base + h * sq.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i <= B_DONE; ++i) mbar_init(bar(i), i == B_P ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t issued = 0;
      mbar_arrive_expect_tx(bar(B_Q), T::Q_BYTES);
      for (int cb = 0; cb < T::CB; ++cb)
        tma_load_3d(base + T::OFF_Q + cb * kQT * 128, &tm_q, cb * 64, h * G, sq.q_off + tok0, bar(B_Q));
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bar(B_EMPTY + s), ((j / NS) & 1) ^ 1, abort_flag)) {
          record_error(a.err, kErrWaitTimeout | 0x11);
          *abort_flag = 1;
          break;
        }
        const uint32_t full = bar(B_FULL + s);
        mbar_arrive_expect_tx(full, T::STAGE);
        const uint32_t st = base + T::OFF_KV + s * T::STAGE;
        const int row = (tile_base + j) * kKT;
        for (int cb = 0; cb < T::CB; ++cb) {
          tma_load_2d(st + cb * kKT * 128, &tm_khi, cb * 64, row, full);
          tma_load_2d(st + T::K_BYTES + cb * kKT * 128, &tm_klo, cb * 64, row, full);
        }
        tma_load_2d(st + 2 * T::K_BYTES, &tm_v, 0, (tile_base + j) * D, full);
        ++issued;
      }
      // no copy may outlive the CTA
      mbar_wait(bar(B_Q), 0, nullptr);
      for (uint32_t j = issued > uint32_t(NS) ? issued - NS : 0; j < issued; ++j)
        mbar_wait(bar(B_FULL + j % NS), (j / NS) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16_f32(kQT, kKT);
      constexpr uint32_t idO = idesc_f16_f32(kQT, D);
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j % NS;
        if (!mbar_wait(bar(B_FULL + s), (j / NS) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t qa = base + T::OFF_Q, ka = base + T::OFF_KV + s * T::STAGE;
        const uint32_t dst = tmem + T::S_COL0 + (j & 1) * kKT;
#pragma unroll
        for (int part = 0; part < 2; ++part) {          // K_hi then K_lo, accumulated
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t qoff = (k >> 2) * kQT * 128 + (k & 3) * 32;
            const uint32_t koff = part * T::K_BYTES + (k >> 2) * kKT * 128 + (k & 3) * 32;
            umma_f16(dst, sdesc_k_sw128(qa + qoff), sdesc_k_sw128(ka + koff), idS, (part | k) != 0);
          }
        }
        umma_commit(bar(B_S + (j & 1)));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bar(B_P), j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pa = base + T::OFF_P, va = base + T::OFF_KV + s * T::STAGE + 2 * T::K_BYTES;
#pragma unroll
        for (int k = 0; k < kKT / 16; ++k)
          umma_f16(tmem + T::O_COL, sdesc_k_sw128(pa + k * 32), sdesc_k_sw128(va + k * 32), idO, (j > 0 || k > 0));
        umma_commit(bar(B_PV));
        umma_commit(bar(B_EMPTY + s));
        if (j + 2 < n_kv) ok = issue_s(j + 2);
      }
      if (!ok) {
        record_error(a.err, kErrWaitTimeout | 0x12);
        *abort_flag = 1;
      }
      // every MMA issued by this thread has completed before TMEM is released
      umma_commit(bar(B_DONE));
      mbar_wait(bar(B_DONE), 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 2..5)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + (uint32_t(quad * 32) << 16);
    const int qpos = qpos0 + row / G;
    float m_used = -INFINITY, l = 0.f;
    uint8_t* P = smem + T::OFF_P;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(bar(B_S + (j & 1)), (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[kKT];
#pragma unroll
      for (int c = 0; c < kKT / 32; ++c) {
        uint32_t r32[32];
        tmem_ld32(lane_addr + T::S_COL0 + (j & 1) * kKT + 32 * c, r32);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 * c + i] = __uint_as_float(r32[i]) * a.scale_log2;
      }
      const int kpos0 = j * kKT;
      float mx = -INFINITY;
      if (kpos0 + kKT - 1 > qpos0) {      // tile reaches past the diagonal of row 0: mask
#pragma unroll
        for (int i = 0; i < kKT; ++i) {
          if (kpos0 + i > qpos) sv[i] = -INFINITY;
          mx = fmaxf(mx, sv[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kKT; ++i) mx = fmaxf(mx, sv[i]);
      }
      // previous P consumed and O stable before either is touched
      if (j > 0 && !mbar_wait(bar(B_PV), (j - 1) & 1, abort_flag)) { ok = false; break; }
      const bool need = mx > m_used + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float mnew = need ? mx : m_used;
        const float alpha = exp2f(m_used - mnew);   // 0 when m_used = -inf
        l *= alpha;
        m_used = mnew;
        if (j > 0) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r32[32];
            tmem_ld32(lane_addr + T::O_COL + 32 * c, r32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(__uint_as_float(r32[i]) * alpha);
            tmem_st32(lane_addr + T::O_COL + 32 * c, r32);
          }
          tmem_wait_st();
        }
      }
      // P = 2^(s - m) in fp16: one K-major 128-byte-swizzled row of 64 tokens
#pragma unroll
      for (int c = 0; c < kKT / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = exp2f(sv[8 * c + 2 * i] - m_used), p1 = exp2f(sv[8 * c + 2 * i + 1] - m_used);
          l += p0 + p1;
          __half2 hp = __floats2half2_rn(p0, p1);
          w[i] = *reinterpret_cast<uint32_t*>(&hp);
        }
        *reinterpret_cast<uint4*>(P + row * 128 + ((c ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_P));
    }
    if (!ok) {
      record_error(a.err, kErrWaitTimeout | 0x13);
      *abort_flag = 1;
    } else if (mbar_wait(bar(B_PV), (n_kv - 1) & 1, abort_flag)) {
      tc_fence_after();
      const int t = tok0 + row / G;
      const float inv = 1.f / l;
      __half* orow = a.out + (int64_t(sq.q_off + t) * b.Hq + h * G + row % G) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r32[32];
        tmem_ld32(lane_addr + T::O_COL + 32 * c, r32);
        tmem_wait_ld();
        if (t < sq.q_len) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __half2 hv = __floats2half2_rn(__uint_as_float(r32[i + 2 * k]) * inv,
                                             __uint_as_float(r32[i + 2 * k + 1]) * inv);
              w[k] = *reinterpret_cast<uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(orow + 32 * c + i) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    } else {
      record_error(a.err, kErrWaitTimeout | 0x14);
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
// Batch sorted by decreasing length (heavy work first), with tile and query-tile offsets.
PrefillBatch plan(const Layout& L, const Batch& in, int n_q_heads, int64_t* n_tiles_total, int64_t* n_qtiles) {
  PrefillBatch b{};
  b.n = in.n;
  b.H = L.n_kv_heads;
  b.G = n_q_heads / L.n_kv_heads;
  b.Hq = n_q_heads;
  std::vector<int> order(in.n);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return in.s[x].a > in.s[y].a; });
  const int TT = kQT / b.G;
  int64_t tiles = 0, qts = 0;
  for (int i = 0; i < in.n; ++i) {
    const SeqDesc& d = in.s[order[i]];
    PrefillSeq& p = b.s[i];
    p.seq_id = d.seq_id;
    p.len = d.a;
    p.q_len = d.b;
    p.q_off = d.c;
    p.tile_base = int32_t(tiles);
    p.n_tiles = (d.a + kKT - 1) / kKT;
    p.qt_begin = int32_t(qts);
    tiles += int64_t(p.n_tiles) * b.H;
    qts += (d.b + TT - 1) / TT;
  }
  *n_tiles_total = tiles;
  *n_qtiles = qts;
  return b;
}

template <int D>
cudaError_t run(const Layout& L, int layer, const Batch& in, int total_q, int n_q_heads, const void* q, void* out,
                float scale, void* ws, cudaStream_t s) {
  int64_t n_tiles = 0, n_qt = 0;
  const PrefillBatch b = plan(L, in, n_q_heads, &n_tiles, &n_qt);
  const int64_t per = n_tiles * kKT * D;
  __half* khi = static_cast<__half*>(ws);
  __half* klo = khi + per;
  __half* vws = klo + per;
  dequant_tiles_kernel<D><<<unsigned(n_tiles), 256, 0, s>>>(L, layer, b, khi, klo, vws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  CUtensorMap mq, mkh, mkl, mv;
  const int G = b.G;
  {
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(n_q_heads), cuuint64_t(total_q)};
    cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(n_q_heads) * D * 2};
    cuuint32_t box[3] = {64, cuuint32_t(G), cuuint32_t(kQT / G)};
    if (!make_tensor_map(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, const_cast<void*>(q), 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(n_tiles) * kKT};
    cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    cuuint32_t box[2] = {64, kKT};
    if (!make_tensor_map(&mkh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, khi, 2, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tensor_map(&mkl, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, klo, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {cuuint64_t(kKT), cuuint64_t(n_tiles) * D};
    cuuint64_t strides[1] = {cuuint64_t(kKT) * 2};
    cuuint32_t box[2] = {64, cuuint32_t(D)};
    if (!make_tensor_map(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, vws, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  using T = PTraits<D>;
  static bool configured = false;
  if (!configured) {
    e = cudaFuncSetAttribute(prefill_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  PrefillArgs a;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<__half*>(out);
  a.err = L.err;
  dim3 grid(unsigned(n_qt), unsigned(b.H));
  prefill_attn_kernel<D><<<grid, T::NT, T::SMEM, s>>>(mq, mkh, mkl, mv, a, b);
  return cudaGetLastError();
}

}  // namespace

size_t prefill_workspace_bytes(const Layout& L, const Batch& b) {
  int64_t tiles = 0;
  for (int i = 0; i < b.n; ++i) tiles += int64_t((b.s[i].a + kKT - 1) / kKT) * L.n_kv_heads;
  return size_t(tiles) * kKT * L.head_dim * 3 * sizeof(__half);   // K_hi, K_lo, V^T
}

cudaError_t launch_prefill(const Layout& L, int layer, const Batch& b, int total_q, int n_q_heads, const void* q,
                           void* out, float scale, void* ws, size_t, int, cudaStream_t s) {
  if (L.head_dim == 128) return run<128>(L, layer, b, total_q, n_q_heads, q, out, scale, ws, s);
  return run<64>(L, layer, b, total_q, n_q_heads, q, out, scale, ws, s);
}

}  // namespace kvq
