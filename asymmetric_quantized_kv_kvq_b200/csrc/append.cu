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
#include "quant_block.cuh"

namespace kvq {
namespace {

__global__ void pt_update_kernel(int32_t* table, const __grid_constant__ PtUpdate u) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < u.n) table[u.idx[i]] = u.val[i];
}

// One thread quantises one 32-element block of one K or V row: it loads the
// block's 64 bytes with four 16-byte loads, takes the block max in registers
// (no shuffles, one scale and one reciprocal per block), rounds the 32 codes on
// the FMA pipe and writes them with 16-byte stores.  A warp covers the 32
// consecutive blocks of 32 / (D / 32) rows of K only or of V only (warps
// alternate), so its loads and stores stay contiguous and its lanes never
// diverge between the 8-bit and the 4-bit code paths.
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
  const int page = L.page_table[int64_t(sd.seq_id) * L.max_pages_per_seq + page_slot(pos / L.page_tokens, sd.ring)];
  if (page < 0 || page >= L.n_pages) {
    record_error(L.err, kErrBadPage);
    return;
  }
  const int r = pos % L.page_tokens;
  uint8_t* hb = L.head_ptr(layer + sd.l, page, h);
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
__global__ void export_kernel(const Layout L, int layer, int seq_id, int ring, int64_t tok0, int64_t n_tok,
                              uint8_t* kc, uint8_t* ks, uint8_t* vc, uint8_t* vs) {
  const int lane = threadIdx.x & 31;
  const int64_t w = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int H = L.n_kv_heads;
  if (w >= n_tok * H) return;
  const int64_t t = w / H;
  const int h = int(w % H);
  const int64_t pos = tok0 + t;
  const int page = L.page_table[int64_t(seq_id) * L.max_pages_per_seq + page_slot(int(pos / L.page_tokens), ring)];
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

cudaError_t launch_export(const Layout& L, int layer, int seq_id, int ring, int64_t tok0, int64_t n_tok, void* kc,
                          void* ks, void* vc, void* vs, cudaStream_t s) {
  const int64_t warps = n_tok * L.n_kv_heads;
  export_kernel<<<unsigned((warps + 7) / 8), 256, 0, s>>>(L, layer, seq_id, ring, tok0, n_tok, static_cast<uint8_t*>(kc),
                                                          static_cast<uint8_t*>(ks), static_cast<uint8_t*>(vc),
                                                          static_cast<uint8_t*>(vs));
  return cudaGetLastError();
}

}  // namespace kvq
