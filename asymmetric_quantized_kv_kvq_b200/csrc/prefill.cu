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
//     dequantised once, in 64-token tiles of a workspace: K as K_hi = fp16(k^)
//     [64 tokens][D] plus the remainder K_lo = k^ - K_hi (fp16 alone would
//     round the x10 outlier key channels by up to 2^-12 relative, which moves
//     the softmax by ~0.2%), stored as e5m2 x 2^8 at head_dim 128 (k^ to
//     ~2^-15) and as fp16 at head_dim 64 (~22 bits), and V transposed
//     [D][64 tokens] in fp16, so both MMAs read K-major operands.
//     (Dequantising inside the attention kernel would redo it for every
//     128-row query tile: a 4096-token chunk with 4 query heads per KV head
//     has 128 of them.)  Positions past the end are zero.
//     The batch runs in waves of (sequences x a range of KV heads) whose
//     dequantised tiles fit a fixed budget (kWaveTiles, ~60 MB at head_dim
//     128): each wave is dequantised into one half of a two-buffer workspace
//     and attended on its own stream, alternating between two internal
//     streams, so the workspace stays bounded (and mostly in L2) whatever the
//     cache length, and the next wave's CTAs fill SMs as the previous wave's
//     finish.
//  2. prefill_attn_kernel: one CTA per (query tile of 128 rows = 128/G tokens
//     x G query heads of one KV head).  Warp 0 streams Q once, then 128-key
//     tiles (two pass-1 tiles) with 2-D / 3-D TMA tensor loads (128-byte
//     swizzle): lane 0 fills a ring of K_hi / K_lo slots, lane 1 a separate
//     ring of V^T slots, so a key slot refills as soon as its scores are done.
//     Warp 1 owns all 512 TMEM columns (a ring of three S buffers, O) and
//     issues the score MMAs, warp 10 the PV MMAs (fp32 accumulators):
//        S_j = Q K_hi,j^T + Q8 K_lo,j^T  (M 128, N 128: D/16 kind::f16 MMAs and, at
//                                         head_dim 128, D/32 kind::f8f6f4 MMAs on e5m2
//                                         operands, Q8 = e5m2(Q 2^-8) converted once
//                                         per CTA by the softmax warps; at head_dim 64
//                                         K_lo is fp16 and Q K_lo^T takes D/16 more)
//        O  += P_j V_j                   (kind::f16, A = P read from TMEM, 8 MMAs per 128 keys).
//     A tcgen05.mma costs roughly the same time for N up to 128, so wide key
//     tiles halve the instruction count of 64-key ones.  Warps 2-9 run the
//     softmax, two per TMEM lane quadrant (one thread per row) taking whole
//     tiles in turn: tile j goes to the warp of parity j % 2, which reads the
//     row's 128 raw scores, takes their max, hands the running max on to the
//     other warp at once (shared memory and a named barrier of the pair), and
//     then computes the exponentials while the other warp reads and reduces
//     tile j + 1, so the MUFU unit is kept busy.  The causal mask is applied in
//     the read: on the chunks that reach past the tile's first row the keys
//     beyond the row's position become -inf and are written back to S, so the
//     exponentials carry no mask.  sigma log2 e is applied with the max
//     subtracted, the online softmax moves the running max only when it
//     grows by more than 2^8 (then O is rescaled in TMEM), and P is stored as
//     fp16 pairs (tcgen05.st) over the first half of its own S buffer, where
//     the PV MMA takes its A operand; the S buffer returns to the score MMAs
//     when that PV is done, three tiles later.  Each warp keeps a partial row
//     sum; at the end the pair joins them, normalises O and stores it.  Every
//     wait is bounded.
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
  int32_t H, G, Hq;     // H = KV heads of this wave, h0 + [0, H)
  int32_t h0;
  PrefillSeq s[kMaxBatch];
};

// Dequantised 64-token tiles per wave: a wave is one or more whole sequences
// with all KV heads, or one sequence with a range of its heads; a single
// (sequence, head) larger than this is a wave of its own.
constexpr int64_t kWaveTiles = 1536;

// Softmax arithmetic of the attention kernel: three-input max, and 2^x by the
// MUFU approximation with subnormal results flushed (p < 2^-126 contributes
// nothing visible once P is rounded to fp16 for the PV MMA).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named CTA barrier between a producing and a consuming warp: the producer
// arrives without waiting once its shared-memory writes are done, the consumer
// waits; `threads` counts both sides.
__device__ __forceinline__ void nbar_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void nbar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// The remainder K_lo = k^ - fp16(k^) enters the scores at head_dim 128 as e5m2
// (2 mantissa bits, scaled by 2^8) against an e5m2 copy of Q scaled by 2^-8,
// through a kind::f8f6f4 MMA (K = 32 per instruction, twice the fp16 rate):
// the correction term is then exact to ~2^-3 of itself, i.e. k^ to ~2^-15.
// At head_dim 64 K_lo stays fp16.
template <int D>
constexpr bool kLo8 = D == 128;
constexpr float kLoScale = 256.f, kQ8Scale = 1.f / 256.f;

// two fp32 -> e5m2 (round to nearest even, saturating to the largest finite);
// `first` lands in the low byte
__device__ __forceinline__ uint32_t e5m2x2(float first, float second) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
  return r;
}

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
                                                            __half* __restrict__ khi, void* __restrict__ klo,
                                                            __half* __restrict__ vws) {
  __shared__ __align__(16) __half vt[kKT][D + 8];
  const int gt = blockIdx.x;
  const int si = find_seq_by(b, gt, true);
  const PrefillSeq sq = b.s[si];
  const int rel = gt - sq.tile_base;
  const int h = b.h0 + rel / sq.n_tiles, j = rel % sq.n_tiles;
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
    for (int i = 0; i < 8; ++i) hi[i] = __float2half_rn(x[i]);
    *reinterpret_cast<uint4*>(khi + tile_off + t * D + e0) = *reinterpret_cast<uint4*>(hi);
    if constexpr (kLo8<D>) {
      // x - fp16(x) is exact in fp32 (x has at most 19 significant bits), and so is the 2^8 scaling
      uint32_t w[2];
#pragma unroll
      for (int i = 0; i < 2; ++i)
        w[i] = e5m2x2((x[4 * i] - __half2float(hi[4 * i])) * kLoScale,
                      (x[4 * i + 1] - __half2float(hi[4 * i + 1])) * kLoScale) |
               (e5m2x2((x[4 * i + 2] - __half2float(hi[4 * i + 2])) * kLoScale,
                       (x[4 * i + 3] - __half2float(hi[4 * i + 3])) * kLoScale) << 16);
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(klo) + tile_off + t * D + e0) = make_uint2(w[0], w[1]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) lo[i] = __float2half_rn(x[i] - __half2float(hi[i]));
      *reinterpret_cast<uint4*>(static_cast<__half*>(klo) + tile_off + t * D + e0) = *reinterpret_cast<uint4*>(lo);
    }
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
constexpr int kKV = 128;     // key / value tokens per stage: N of S, K of P V (two pass-1 tiles)

template <int D>
struct PTraits {
  static constexpr int CB = D / 64;                      // 128-byte column blocks of a Q / K row
  static constexpr int Q_BYTES = kQT * D * 2;            // CB blocks of [128 rows][128 B]
  static constexpr int K_BYTES = kKV * D * 2;            // CB blocks of [128 rows][128 B]
  static constexpr int V_BYTES = D * kKV * 2;            // two blocks (64 tokens each) of [D rows][128 B]
  static constexpr bool LO8 = kLo8<D>;
  static constexpr int KLO_BYTES = LO8 ? kKV * D : K_BYTES;   // e5m2: one block of [128 rows][128 B]
  static constexpr int Q8_BYTES = LO8 ? kQT * D : 0;          // e5m2 copy of Q, [128 rows][128 B]
  static constexpr int KSLOT = K_BYTES + KLO_BYTES;      // K_hi, K_lo of one 128-key tile
  static constexpr int NSTAGE = D == 128 ? 2 : 3;        // slots of each ring (keys and values separately,
                                                         // so a key slot is refilled as soon as S is done)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_Q8 = OFF_Q + Q_BYTES;
  static constexpr int OFF_K = OFF_Q8 + Q8_BYTES;
  static constexpr int OFF_V = OFF_K + NSTAGE * KSLOT;
  static constexpr int OFF_BAR = OFF_V + NSTAGE * V_BYTES;
  // + alignment slack; never less than ~116 KB so that a second CTA cannot
  // share the SM and wait in tcgen05.alloc
  static constexpr int SMEM_NEED = OFF_BAR + 256 + (128 + 4 * 128) * 4 + 1024;   // barriers, TMEM slot, row (m, l)
  static constexpr int SMEM = SMEM_NEED > 118 * 1024 ? SMEM_NEED : 118 * 1024;
  static constexpr int NT = 352;                         // 11 warps: copies, score MMAs, 2 x 4 softmax, PV MMAs
  static constexpr uint32_t TMEM_COLS = 512;
  // S ring of three 128-column buffers [0, 384) (fp32 scores of 128 keys; P_j is written over the first
  // 64 columns of its own S_j as fp16 pairs once the scores are in registers), O [384, 384 + D)
  static constexpr int NSB = 3;
  static constexpr uint32_t S_COL0 = 0, O_COL = NSB * kKV;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM");
  static_assert(OFF_Q8 % 1024 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && KSLOT % 1024 == 0 &&
                    K_BYTES % 1024 == 0 && V_BYTES % 1024 == 0,
                "swizzle atoms");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct PrefillArgs {
  float scale_log2;
  __half* out;
  uint32_t* err;
};

template <int D>
__global__ void __launch_bounds__(352, 1)
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
  // barriers: q_full | k_full[NS] | k_empty[NS] | v_full[NS] | v_empty[NS] | s_full[3] | p_full[3] | pv_done[3]
  // | done | done2 | q8; S, P and PV have one barrier per buffer of the S ring (tile j uses buffer j % 3;
  // pv_done of a buffer also frees it for the scores three tiles later)
  constexpr int NSB = T::NSB;
  constexpr int B_Q = 0, B_KFULL = 1, B_KEMPTY = 1 + NS, B_VFULL = 1 + 2 * NS, B_VEMPTY = 1 + 3 * NS,
                B_S = 1 + 4 * NS, B_P = B_S + NSB, B_PV = B_P + NSB, B_DONE = B_PV + NSB, B_DONE2 = B_DONE + 1,
                B_Q8 = B_DONE2 + 1;
  static_assert(B_Q8 < 28, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 28);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 29);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int si = find_seq_by(b, blockIdx.x, false);
  const PrefillSeq sq = b.s[si];
  const int G = b.G, TT = kQT / G;                        // tokens per query tile
  const int nq = (sq.q_len + TT - 1) / TT;
  const int qt = nq - 1 - (int(blockIdx.x) - sq.qt_begin); // heavy tiles first
  const int h = b.h0 + blockIdx.y;                        // KV head
  const int tok0 = qt * TT;                                // first chunk row of this tile
  const int qpos0 = sq.len - sq.q_len + tok0;              // absolute position of row 0
  const int qpos_last = sq.len - sq.q_len + min(tok0 + TT, sq.q_len) - 1;
  const int n_kv = qpos_last / kKV + 1;
  const int tile_base = sq.tile_base + blockIdx.y * sq.n_tiles;   // first 64-token pass-1 tile of this head

  if (threadIdx.x == 0) {
    for (int i = 0; i <= B_Q8; ++i)
      mbar_init(bar(i), (i >= B_P && i < B_P + NSB) ? 128u : i == B_Q8 ? 256u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers: lane 0 Q and keys, lane 1 values
    if (lane == 0) {
      uint32_t issued = 0;
      mbar_arrive_expect_tx(bar(B_Q), T::Q_BYTES);
      for (int cb = 0; cb < T::CB; ++cb)
        tma_load_3d(base + T::OFF_Q + cb * kQT * 128, &tm_q, cb * 64, h * G, sq.q_off + tok0, bar(B_Q));
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bar(B_KEMPTY + s), ((j / NS) & 1) ^ 1, abort_flag)) {
          record_error(a.err, kErrWaitTimeout | 0x11);
          *abort_flag = 1;
          break;
        }
        const uint32_t full = bar(B_KFULL + s);
        mbar_arrive_expect_tx(full, T::KSLOT);
        const uint32_t st = base + T::OFF_K + s * T::KSLOT;
        const int t64 = tile_base + 2 * j;                   // two consecutive pass-1 tiles
        for (int cb = 0; cb < T::CB; ++cb) {
          tma_load_2d(st + cb * kKV * 128, &tm_khi, cb * 64, t64 * 64, full);
          if (!T::LO8) tma_load_2d(st + T::K_BYTES + cb * kKV * 128, &tm_klo, cb * 64, t64 * 64, full);
        }
        if (T::LO8) tma_load_2d(st + T::K_BYTES, &tm_klo, 0, t64 * 64, full);
        ++issued;
      }
      // no copy may outlive the CTA
      mbar_wait(bar(B_Q), 0, nullptr);
      for (uint32_t j = issued > uint32_t(NS) ? issued - NS : 0; j < issued; ++j)
        mbar_wait(bar(B_KFULL + j % NS), (j / NS) & 1, nullptr);
    } else if (lane == 1) {
      uint32_t issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bar(B_VEMPTY + s), ((j / NS) & 1) ^ 1, abort_flag)) {
          record_error(a.err, kErrWaitTimeout | 0x15);
          *abort_flag = 1;
          break;
        }
        const uint32_t full = bar(B_VFULL + s);
        mbar_arrive_expect_tx(full, T::V_BYTES);
        const uint32_t st = base + T::OFF_V + s * T::V_BYTES;
        const int t64 = tile_base + 2 * j;
        tma_load_2d(st, &tm_v, 0, t64 * D, full);
        tma_load_2d(st + D * 128, &tm_v, 0, (t64 + 1) * D, full);
        ++issued;
      }
      for (uint32_t j = issued > uint32_t(NS) ? issued - NS : 0; j < issued; ++j)
        mbar_wait(bar(B_VFULL + j % NS), (j / NS) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score MMAs
    // A tcgen05.mma keeps its issuing thread busy for ~100 cycles whatever its shape (measured), so the
    // score MMAs and the PV MMAs are issued by two warps; they touch disjoint TMEM columns.
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16_f32(kQT, kKV);
      constexpr uint32_t idS8 = idesc_e5m2_f32(kQT, kKV);
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
      const uint64_t qd0 = sdesc_k_sw128(base + T::OFF_Q);
      const uint64_t q8d0 = sdesc_k_sw128(base + T::OFF_Q8);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % NS;
        // S buffer j % 3 held P_(j-3), read by PV(j - 3); the key slot is full
        if (j >= NSB) ok = mbar_wait(bar(B_PV + j % NSB), ((j - NSB) / NSB) & 1, abort_flag);
        if (ok) ok = mbar_wait(bar(B_KFULL + s), (j / NS) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t kd0 = sdesc_k_sw128(base + T::OFF_K + s * T::KSLOT);
        const uint32_t dst = tmem + T::S_COL0 + (j % NSB) * kKV;
        if constexpr (T::LO8) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {          // Q K_hi^T (fp16)
            const uint32_t qoff = (k >> 2) * kQT * 128 + (k & 3) * 32;
            const uint32_t koff = (k >> 2) * kKV * 128 + (k & 3) * 32;
            umma_f16(dst, qd0 + (qoff >> 4), kd0 + (koff >> 4), idS, k != 0);
          }
          // + Q8 K_lo8^T (e5m2, 32 elements = 32 B per MMA); Q8 is written by the softmax warps once
          if (j == 0 && !mbar_wait(bar(B_Q8), 0, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            umma_f8(dst, q8d0 + ((k * 32) >> 4), kd0 + ((T::K_BYTES + k * 32) >> 4), idS8, 1);
        } else {
#pragma unroll
          for (int part = 0; part < 2; ++part) {        // K_hi then K_lo, accumulated
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t qoff = (k >> 2) * kQT * 128 + (k & 3) * 32;
              const uint32_t koff = part * T::K_BYTES + (k >> 2) * kKV * 128 + (k & 3) * 32;
              umma_f16(dst, qd0 + (qoff >> 4), kd0 + (koff >> 4), idS, (part | k) != 0);
            }
          }
        }
        umma_commit(bar(B_S + j % NSB));
        umma_commit(bar(B_KEMPTY + s));                 // the key slot refills once S_j is done
      }
      if (!ok) {
        record_error(a.err, kErrWaitTimeout | 0x12);
        *abort_flag = 1;
      }
      // every MMA issued by this thread has completed before TMEM is released
      umma_commit(bar(B_DONE));
      mbar_wait(bar(B_DONE), 0, nullptr);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ PV MMAs
    if (lane == 0) {
      constexpr uint32_t idO = idesc_f16_f32(kQT, D);
      bool ok = true;
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bar(B_P + j % NSB), (j / NSB) & 1, abort_flag) ||
            !mbar_wait(bar(B_VFULL + s), (j / NS) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // O += P V: A = P in TMEM (16 keys = 8 columns per step), B = V^T [D][128 keys] in two 64-key blocks
        const uint32_t pa = tmem + T::S_COL0 + (j % NSB) * kKV;   // P_j over S_j
        const uint64_t vd0 = sdesc_k_sw128(base + T::OFF_V + s * T::V_BYTES);
#pragma unroll
        for (int k = 0; k < kKV / 16; ++k)
          umma_f16_ta(tmem + T::O_COL, pa + 8 * k, vd0 + (((k >> 2) * D * 128 + (k & 3) * 32) >> 4), idO,
                      (j > 0 || k > 0));
        umma_commit(bar(B_PV + j % NSB));
        umma_commit(bar(B_VEMPTY + s));
      }
      if (!ok) {
        record_error(a.err, kErrWaitTimeout | 0x16);
        *abort_flag = 1;
      }
      umma_commit(bar(B_DONE2));
      mbar_wait(bar(B_DONE2), 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 2..9)
    // Two warps per TMEM lane quadrant (one thread per row) take turns: the warp of parity `par` runs
    // the whole 128-key tiles j with j % 2 == par.  The running row max m passes from tile j to tile
    // j + 1 through shared memory at a named barrier of the quadrant's two warps (arrive after
    // writing, wait before reading), and is handed on as soon as the tile's max is known, so one
    // warp's exponentials (the MUFU unit) overlap the other's TMEM read and max of the next tile.
    // Each warp keeps its own partial row sum l against its own last m; the two are joined at the end.
    constexpr int BAR_L = 9, NTH = 256;
    const int quad = warp & 3, par = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + (uint32_t(quad * 32) << 16);
    const int qpos = qpos0 + row / G;
    const int bar_from = 1 + quad + 4 * (par ^ 1), bar_to = 1 + quad + 4 * par;   // named barriers 1..8
    float* mrow = reinterpret_cast<float*>(bars + 32);   // [128 rows]: m of the latest tile
    float* fin_ml = mrow + 128;                          // [2 parities][m, l][128 rows]
    float m_own = -INFINITY, l_own = 0.f;
    bool wok = true;
    if constexpr (T::LO8) {
      // Q8 = e5m2(Q 2^-8): thread (row r, half hf) converts elements [64 hf, 64 hf + 64) of row r from
      // the fp16 tile (column block hf, 128-byte swizzle) into the e5m2 tile (one column block)
      const int st = threadIdx.x - 64, r = st >> 1, hf = st & 1;
      if (mbar_wait(bar(B_Q), 0, abort_flag)) {
        const uint8_t* src = smem + T::OFF_Q + hf * kQT * 128 + r * 128;
        uint8_t* dq = smem + T::OFF_Q8 + r * 128;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 w = *reinterpret_cast<const uint4*>(src + ((c8 ^ (r & 7)) << 4));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          uint32_t o[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float2 f0 = h2_to_f2(ws[2 * i]), f1 = h2_to_f2(ws[2 * i + 1]);
            o[i] = e5m2x2(f0.x * kQ8Scale, f0.y * kQ8Scale) | (e5m2x2(f1.x * kQ8Scale, f1.y * kQ8Scale) << 16);
          }
          const int x = 64 * hf + 8 * c8;                         // byte = element index in the e5m2 row
          *reinterpret_cast<uint2*>(dq + ((((x >> 4) ^ (r & 7)) << 4) | (x & 8))) = make_uint2(o[0], o[1]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
      mbar_arrive(bar(B_Q8));
    }
    for (int j = par; j < n_kv; j += 2) {
      const int sb = j % NSB;
      wok = wok && __all_sync(0xffffffffu, mbar_wait(bar(B_S + sb), (j / NSB) & 1, abort_flag));
      const uint32_t sbuf = lane_addr + T::S_COL0 + sb * kKV;
      const int kpos0 = j * kKV;
      // pass 1: the row's 128 raw scores and their max (sigma log2 e > 0 keeps the order).  Only
      // 32-key chunks that reach past the first row's position need the causal mask: there the
      // keys past the row's position are set to -inf and the chunk is written back to S, so that
      // the exponentials (2^-inf = 0) need no mask on any tile
      float mx = -INFINITY;
      if (wok) {
        tc_fence_after();
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        bool wrote = false;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // two reads of 64 keys
          uint32_t sv[64];
          tmem_ld32(sbuf + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(sbuf + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * hh + cc;
            if (kpos0 + 32 * c + 31 > qpos0) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float v = kpos0 + 32 * c + i <= qpos ? __uint_as_float(sv[32 * cc + i]) : -INFINITY;
                sv[32 * cc + i] = __float_as_uint(v);
                mq[i & 3] = fmaxf(mq[i & 3], v);
              }
              tmem_st32(sbuf + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * cc]));
              wrote = true;
            } else {
              // four independent three-input max chains (a short dependency chain)
#pragma unroll
              for (int i = 0; i < 32; i += 8)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  mq[q] = fmax3(mq[q], __uint_as_float(sv[32 * cc + i + 2 * q]),
                                __uint_as_float(sv[32 * cc + i + 2 * q + 1]));
            }
          }
        }
        mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
        if (wrote) tmem_wait_st();                   // the masked chunks are in S before pass 2 reads them
      }
      mx *= a.scale_log2;
      // the running max after tile j - 1, from the quadrant's other warp
      float m_prev = -INFINITY;
      if (j > 0) {
        nbar_sync(bar_from, 64);
        m_prev = mrow[row];
      }
      // lazy max: m moves only when the tile's max exceeds it by more than 2^8 (p <= 2^8 fits fp16)
      const bool need = mx > m_prev + 8.f;
      const float m_used = need ? mx : m_prev;
      if (j + 1 < n_kv) {
        mrow[row] = m_used;
        nbar_arrive(bar_to, 64);
      }
      if (m_used != m_own) {   // this warp's partial sum follows the new m (0 while it has none)
        l_own *= exp2f(m_own - m_used);
        m_own = m_used;
      }
      if (__any_sync(0xffffffffu, need) && j > 0) {
        // O holds every PV up to PV(j - 1) at m_prev: rescale it once PV(j - 1) is done, before
        // P_j is released (PV(j) follows in the PV warp's order)
        const float alpha = exp2f(m_prev - m_used);   // 0 when m_prev = -inf, 1 where m stays
        wok = wok && __all_sync(0xffffffffu, mbar_wait(bar(B_PV + (j - 1) % NSB), ((j - 1) / NSB) & 1, abort_flag));
        if (wok) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r32[32];
            const uint32_t oc = lane_addr + T::O_COL + 32 * c;
            tmem_ld32(oc, r32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(__uint_as_float(r32[i]) * alpha);
            tmem_st32(oc, r32);
          }
          tmem_wait_st();
        }
      }
      // pass 2: P = 2^(sigma log2 e s - m) as fp16 pairs over the first 64 columns of S_j: the scores
      // are read again 32 keys at a time, the next chunk's read in flight while one is processed (P of
      // chunk c lands in columns [16c, 16c + 16), whose scores are already in registers); pairs: one
      // f32x2 FMA scales and shifts two scores, one f32x2 add sums two p
      if (!wok) *abort_flag = 1;
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_used, -m_used);
      float2 l2 = make_float2(0.f, 0.f);
      uint32_t sv[2][32];
      if (wok) {
        tmem_ld32(sbuf, sv[0]);
        tmem_wait_ld();
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (wok && c < 3) tmem_ld32(sbuf + 32 * (c + 1), sv[(c + 1) & 1]);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 x = ffma2(make_float2(__uint_as_float(sv[c & 1][2 * i]),
                                             __uint_as_float(sv[c & 1][2 * i + 1])), sc2, nm2);
          const float p0 = ex2_ftz(x.x);   // 0 for a masked key (-inf)
          const float p1 = ex2_ftz(x.y);
          l2 = fadd2(l2, make_float2(p0, p1));
          __half2 hp = __floats2half2_rn(p0, p1);
          pk[i] = *reinterpret_cast<uint32_t*>(&hp);
        }
        if (wok) {
          tmem_st16(sbuf + 16 * c, pk);
          if (c < 3) tmem_wait_ld();
        }
      }
      l_own += l2.x + l2.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_P + sb));
    }
    // the (m, l) of both warps of each row; every softmax thread takes part, so the exit is uniform
    fin_ml[(2 * par) * 128 + row] = m_own;
    fin_ml[(2 * par + 1) * 128 + row] = l_own;
    bool fin = wok && __all_sync(0xffffffffu, mbar_wait(bar(B_PV + (n_kv - 1) % NSB), ((n_kv - 1) / NSB) & 1,
                                                      abort_flag));
    fin = bar_red_and(BAR_L, NTH, fin);
    if (!fin) {
      record_error(a.err, kErrWaitTimeout | 0x13);
      *abort_flag = 1;
    } else {
      // O is at the last tile's m, the larger of the two warps' m
      const float mo = fin_ml[(2 * (par ^ 1)) * 128 + row], lo = fin_ml[(2 * (par ^ 1) + 1) * 128 + row];
      const float mf = fmaxf(m_own, mo);
      const float l = (m_own == mf ? l_own : l_own * exp2f(m_own - mf)) + (mo == mf ? lo : lo * exp2f(mo - mf));
      tc_fence_after();
      const int t = tok0 + row / G;
      const float inv = 1.f / l;
      __half* orow = a.out + (int64_t(sq.q_off + t) * b.Hq + h * G + row % G) * D + (D / 2) * par;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r32[32];
        tmem_ld32(lane_addr + T::O_COL + (D / 2) * par + 32 * c, r32);
        tmem_wait_ld();
        if (t < sq.q_len) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __half2 hv = __floats2half2_rn(__uint_as_float(r32[i + 2 * k]) * inv,
                                             __uint_as_float(r32[i + 2 * k + 1]) * inv);
              w4[k] = *reinterpret_cast<uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(orow + 32 * c + i) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
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
// Sequence order: decreasing length (heavy work first).
std::vector<int> length_order(const Batch& in) {
  std::vector<int> order(in.n);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return in.s[x].a > in.s[y].a; });
  return order;
}

struct Wave {
  int first, count;     // positions in the length order
  int h0, nh;           // KV heads
  int64_t tiles;
};

// Waves over the length order: consecutive whole sequences while they fit kWaveTiles,
// a sequence that does not fit alone split into head ranges.
std::vector<Wave> make_waves(const Batch& in, const std::vector<int>& order, int H) {
  std::vector<Wave> w;
  auto tiles_of = [&](int i) { return int64_t((in.s[order[i]].a + kKT - 1) / kKT); };
  int i = 0;
  while (i < in.n) {
    const int64_t t0 = tiles_of(i);
    if (t0 * H > kWaveTiles) {
      const int nh = int(std::max<int64_t>(1, std::min<int64_t>(H, kWaveTiles / t0)));
      for (int h0 = 0; h0 < H; h0 += nh) {
        const int n = std::min(nh, H - h0);
        w.push_back({i, 1, h0, n, t0 * n});
      }
      ++i;
      continue;
    }
    Wave v{i, 0, 0, H, 0};
    while (i < in.n && v.tiles + tiles_of(i) * H <= kWaveTiles) {
      v.tiles += tiles_of(i) * H;
      ++v.count;
      ++i;
    }
    w.push_back(v);
  }
  return w;
}

// Batch of one wave, with tile and query-tile offsets.
PrefillBatch plan(const Batch& in, const std::vector<int>& order, const Wave& v, int H, int n_q_heads,
                  int64_t* n_tiles_total, int64_t* n_qtiles) {
  PrefillBatch b{};
  b.n = v.count;
  b.H = v.nh;
  b.h0 = v.h0;
  b.G = n_q_heads / H;
  b.Hq = n_q_heads;
  const int TT = kQT / b.G;
  int64_t tiles = 0, qts = 0;
  for (int i = 0; i < v.count; ++i) {
    const SeqDesc& d = in.s[order[v.first + i]];
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

// Tiles of the largest wave among those that alternate into workspace half k (waves k, k + 2, ...).
int64_t half_tiles(const std::vector<Wave>& w, int k) {
  int64_t m = 0;
  for (size_t i = k; i < w.size(); i += 2) m = std::max(m, w[i].tiles);
  return m;
}

// One wave: dequantise into ws, then the attention kernel, on stream s.
template <int D>
cudaError_t run_wave(const Layout& L, int layer, const PrefillBatch& b, int64_t n_tiles, int64_t n_qt,
                     const CUtensorMap& mq, const void* out, float scale, void* ws, cudaStream_t s) {
  const int64_t per = n_tiles * kKT * D;
  __half* khi = static_cast<__half*>(ws);
  __half* klo = khi + per;          // fp16 [tokens][D], or e5m2 [tokens][D] in its first half (head_dim 128)
  __half* vws = klo + per;
  dequant_tiles_kernel<D><<<unsigned(n_tiles), 256, 0, s>>>(L, layer, b, khi, klo, vws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mkh, mkl, mv;
  {
    cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(n_tiles) * kKT};
    cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    cuuint32_t box[2] = {64, kKV};
    if (!make_tensor_map(&mkh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, khi, 2, dims, strides, box)) return cudaErrorInvalidValue;
    if (kLo8<D>) {
      cuuint64_t strides8[1] = {cuuint64_t(D)};
      cuuint32_t box8[2] = {cuuint32_t(D), kKV};
      if (!make_tensor_map(&mkl, CU_TENSOR_MAP_DATA_TYPE_UINT8, klo, 2, dims, strides8, box8)) return cudaErrorInvalidValue;
    } else if (!make_tensor_map(&mkl, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, klo, 2, dims, strides, box)) {
      return cudaErrorInvalidValue;
    }
  }
  {
    cuuint64_t dims[2] = {cuuint64_t(kKT), cuuint64_t(n_tiles) * D};
    cuuint64_t strides[1] = {cuuint64_t(kKT) * 2};
    cuuint32_t box[2] = {64, cuuint32_t(D)};
    if (!make_tensor_map(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, vws, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  using T = PTraits<D>;
  PrefillArgs a;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<__half*>(const_cast<void*>(out));
  a.err = L.err;
  dim3 grid(unsigned(n_qt), unsigned(b.H));
  prefill_attn_kernel<D><<<grid, T::NT, T::SMEM, s>>>(mq, mkh, mkl, mv, a, b);
  return cudaGetLastError();
}

template <int D>
cudaError_t run(const Layout& L, int layer, const Batch& in, int total_q, int n_q_heads, const void* q, void* out,
                float scale, void* ws, const PrefillStreams& ps, cudaStream_t s) {
  const int H = L.n_kv_heads, G = n_q_heads / H;
  const std::vector<int> order = length_order(in);
  const std::vector<Wave> waves = make_waves(in, order, H);
  CUtensorMap mq;
  {
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(n_q_heads), cuuint64_t(total_q)};
    cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(n_q_heads) * D * 2};
    cuuint32_t box[3] = {64, cuuint32_t(G), cuuint32_t(kQT / G)};
    if (!make_tensor_map(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, const_cast<void*>(q), 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  using T = PTraits<D>;
  static bool configured = false;
  if (!configured) {
    const cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const size_t half_bytes = size_t(half_tiles(waves, 0)) * kKT * D * 3 * sizeof(__half);   // start of half 1
  if (waves.size() == 1) {
    int64_t nt = 0, nq = 0;
    const PrefillBatch b = plan(in, order, waves[0], H, n_q_heads, &nt, &nq);
    return run_wave<D>(L, layer, b, nt, nq, mq, out, scale, ws, s);
  }
  // several waves: alternate two internal streams and two workspace halves; the caller's
  // stream is forked to both and joined back, so the call stays ordered (and capturable)
  cudaError_t e = cudaEventRecord(ps.fork, s);
  for (int k = 0; k < 2 && e == cudaSuccess; ++k) e = cudaStreamWaitEvent(ps.s[k], ps.fork, 0);
  for (size_t w = 0; w < waves.size() && e == cudaSuccess; ++w) {
    int64_t nt = 0, nq = 0;
    const PrefillBatch b = plan(in, order, waves[w], H, n_q_heads, &nt, &nq);
    void* half = static_cast<uint8_t*>(ws) + (w & 1) * half_bytes;
    e = run_wave<D>(L, layer, b, nt, nq, mq, out, scale, half, ps.s[w & 1]);
  }
  for (int k = 0; k < 2; ++k) {
    const cudaError_t e2 = cudaEventRecord(ps.join[k], ps.s[k]);
    if (e == cudaSuccess) e = e2;
    const cudaError_t e3 = cudaStreamWaitEvent(s, ps.join[k], 0);
    if (e == cudaSuccess) e = e3;
  }
  return e;
}

}  // namespace

size_t prefill_workspace_bytes(const Layout& L, const Batch& b) {
  const std::vector<Wave> waves = make_waves(b, length_order(b), L.n_kv_heads);
  // K_hi, K_lo, V^T: half 0 holds the largest even-numbered wave, half 1 the largest odd-numbered one
  return size_t(half_tiles(waves, 0) + half_tiles(waves, 1)) * kKT * L.head_dim * 3 * sizeof(__half);
}

cudaError_t launch_prefill(const Layout& L, int layer, const Batch& b, int total_q, int n_q_heads, const void* q,
                           void* out, float scale, void* ws, size_t, const PrefillStreams& ps, cudaStream_t s) {
  if (L.head_dim == 128) return run<128>(L, layer, b, total_q, n_q_heads, q, out, scale, ws, ps, s);
  return run<64>(L, layer, b, total_q, n_q_heads, q, out, scale, ws, ps, s);
}

}  // namespace kvq
