// Arguments and work decomposition shared by the split-KV decode kernels: the
// flat list of (sequence, KV head, chunk) units is cut into equal contiguous
// ranges, one per CTA ("stream-K"); a CTA walks its range segment by segment,
// a segment being the chunks of one (sequence, KV head) item inside the range.
#pragma once

#include <cuda_fp16.h>

#include "kvq_internal.cuh"
#include "sm100_util.cuh"

namespace kvq {

struct DecodeArgs {
  Layout L;
  int layer;
  int n_q_heads;
  const __half* q;
  __half* out;
  float* ws_o;        // [slots][G][D]
  float* ws_ml;       // [slots][G][2]
  float scale_log2;   // sigma * log2(e)
  int64_t total_chunks;
  int64_t cpc;        // chunks per CTA
  int chunk;          // tokens per work chunk: gcd(C, page_tokens) <= C, so a chunk never crosses a page
};

struct DecodeSeg {
  int bi, h, k0, n;   // n: chunks holding tokens to process (0 inside an item's padding)
  int adv;            // flat positions the segment covers (n plus the padding after it)
};

// Segment of the flat chunk list starting at x: (sequence, head, first chunk, count).  An
// item may be padded to a whole number of CTA ranges, so that no range crosses an item; the
// padded chunks hold no tokens and are skipped (n counts only the real ones, adv all).
__device__ __forceinline__ DecodeSeg decode_find_seg(const Batch& b, int64_t x, int64_t x1) {
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.s[mid].b <= x) lo = mid; else hi = mid - 1;
  }
  const int nch = b.s[lo].c;
  const int64_t rel = x - b.s[lo].b;
  const int h = int(rel / nch);
  const int k0 = int(rel - int64_t(h) * nch);
  const int64_t item_end = b.s[lo].b + int64_t(h + 1) * nch;
  const int adv = int((x1 < item_end ? x1 : item_end) - x);
  const int real = b.s[lo].cr > 0 ? b.s[lo].cr : nch;
  const int n = real - k0 < adv ? (real - k0 > 0 ? real - k0 : 0) : adv;
  return {lo, h, k0, n, adv};
}

// ---- value codes on CUDA cores ------------------------------------------------
// PV lane `vs` owns 8 elements of the row: element index of value i (0..7).
template <int VB>
__device__ __forceinline__ int v_elem(int vs, int i) {
  if (VB == 4) return 32 * (vs >> 2) + 4 * (vs & 3) + (i < 4 ? i : i + 12);
  return 8 * vs + i;
}
template <int VB>
__device__ __forceinline__ int v_block(int vs) {
  return VB == 16 ? 0 : (vs >> 2);
}

template <int VB>
__device__ __forceinline__ void load_v8(const uint8_t* row, int vs, float2 (&vf)[4]) {
  if (VB == 4) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(row + 4 * vs);
    cvt_u4x4(w & 0x0F0F0F0Fu, vf[0], vf[1]);
    cvt_u4x4((w >> 4) & 0x0F0F0F0Fu, vf[2], vf[3]);
  } else if (VB == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 8 * vs);
    cvt_s8x4(w.x, vf[0], vf[1]);
    cvt_s8x4(w.y, vf[2], vf[3]);
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * vs);
    vf[0] = h2_to_f2(w.x); vf[1] = h2_to_f2(w.y); vf[2] = h2_to_f2(w.z); vf[3] = h2_to_f2(w.w);
  }
}

}  // namespace kvq
