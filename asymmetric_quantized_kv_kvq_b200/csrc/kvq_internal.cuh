// Internal definitions shared by the host library and the sm_100a kernels.
//
// HBM layout of the page pool (one cudaMalloc per cache):
//   pool[layer][page][kv_head] -> one "head block" of page_tokens tokens:
//     K codes  [P][k_row]   int8 (8-bit) | packed nibbles (4-bit, D/2 B) | fp16 (16-bit)
//     K scales [P][D/32]    fp16                     (absent for 16-bit)
//     V codes  [P][v_row]
//     V scales [P][D/32]    fp16                     (absent for 16-bit)
//   Every sub-array is a multiple of 16 B (page_tokens is a multiple of 64), so
//   a token range of one sub-array is one 16-B aligned bulk copy, and the head
//   block holds exactly page_tokens * (K + V bytes per token): the footprint is
//   the closed form of the KVSplit page's memory table with no padding.
//   Rows are token-major and in canonical block order, so exporting a token
//   range is a plain gather by page.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int QK = 32;                 // elements per quantisation block
constexpr int kMaxBatch = KVQ_MAX_BATCH;

// Device error codes (first one recorded wins; read by kvq_cache_check).
enum : uint32_t {
  kErrNone = 0,
  kErrWaitTimeout = 0x100,             // | barrier id: an mbarrier wait exceeded its limit
  kErrBadPage = 0x200,                 // a page-table entry was unmapped or out of range
  kErrBadIndex = 0x300,
};

struct Layout {
  uint8_t* pool;
  const int32_t* page_table;           // [max_seqs][max_pages_per_seq], -1 = unmapped
  uint32_t* err;                       // device error word
  int64_t head_block;                  // bytes per (layer, page, head)
  int32_t n_layers;
  int32_t n_pages;                     // pages in the pool
  int32_t max_pages_per_seq;
  int32_t n_kv_heads;
  int32_t page_tokens;
  int32_t head_dim;
  int32_t k_bits, v_bits;
  int32_t k_row, v_row;                // code bytes per token
  int32_t s_row;                       // scale bytes per token (D/32 * 2), 0 for 16-bit
  int32_t k_scales_off, v_codes_off, v_scales_off;   // byte offsets inside a head block
  int32_t decode_tc;                   // KVQ_CACHE_DECODE_TENSOR_CORES was set
  int32_t* counters;                   // [kMaxBatch * n_kv_heads] split-item counters of the decode kernel (zero at rest)
  uint64_t wait_ns;                    // limit of every bounded wait of the decode kernel
  int32_t test_withhold;               // test hook: the decode kernel withholds one stage's arrival

  __host__ __device__ __forceinline__ uint8_t* head_ptr(int layer, int page, int head) const {
    return pool + ((int64_t(layer) * n_pages + page) * n_kv_heads + head) * head_block;
  }
};

inline int code_row_bytes(int bits, int D) { return bits == 16 ? 2 * D : bits == 8 ? D : D / 2; }

// One sequence of a batched call.  Field meaning depends on the operation:
//   append : a = first position written (len - n_new), b = n_new, c = row offset in k/v
//   decode : a = len, b = flat chunk offset of the sequence's first item, c = chunks per item,
//            lo = first position attended (len - window for a rotating window, else 0)
//   prefill: a = len, b = q_len, c = row offset in q/out
// ring: page-table slots of a rotating-window sequence (logical page p lives in
// slot p % ring), 0 for a linear page table.
// l: layer of the entry, counted from the launch's layer (append and decode):
// a layer-batched call lists every (layer, sequence) pair as an entry of one
// launch; the layers of one launch share a format, so layer l's head blocks lie
// l * n_pages * n_kv_heads head blocks past the launch layer's.
struct SeqDesc {
  int32_t seq_id;
  int32_t a, b, c;
  int32_t lo, ring;
  int32_t cr;   // decode: chunks per head that hold tokens (c may be padded past them; 0 = c)
  int32_t l;
};

// Page-table slot of logical page p of a sequence.
__host__ __device__ __forceinline__ int page_slot(int p, int ring) { return ring ? p % ring : p; }

struct Batch {
  int32_t n;
  SeqDesc s[kMaxBatch];
};

// Page-table update: entries (index into the table, value), applied in order.
constexpr int kMaxPtUpdates = 1024;
struct PtUpdate {
  int32_t n;
  int32_t idx[kMaxPtUpdates];
  int32_t val[kMaxPtUpdates];
};

// Page deduplication: one layer's pool region (page i starts at base + i * bytes,
// bytes = n_kv_heads head blocks) and page lists passed by value to the kernels.
constexpr int kDedupBatch = 1024;    // pages (or pairs) per launch
constexpr int kDedupLayers = 256;    // layers per launch (more layers: several launches, sums add up)
struct PageRegion {
  const uint8_t* base;
  int64_t bytes;
};
struct PageList {
  int32_t n;
  int32_t page[kDedupBatch];
  PageRegion layer[kDedupLayers];
};
struct PagePairs {
  int32_t n;
  int32_t a[kDedupBatch], b[kDedupBatch];
  PageRegion layer[kDedupLayers];
};
// hashes: uint32 [n][4] accumulated over launches (zeroed first when asked); diff: uint32 [n],
// nonzero where a pair differs (OR-ed over launches).
cudaError_t launch_page_hash(const PageList& pl, int n_layers, uint32_t* hashes, bool zero_first, cudaStream_t s);
cudaError_t launch_page_compare(const PagePairs& pp, int n_layers, uint32_t* diff, bool zero_first, cudaStream_t s);

__device__ __forceinline__ void record_error(uint32_t* err, uint32_t code) {
  atomicCAS(err, 0u, code);
}

// Sets the text kvq_last_error() returns on this thread; returns `s`.
kvq_status set_last_error(kvq_status s, const char* msg);

// For calls that launch work: KVQ_ERR_UNSUPPORTED for a host-only cache,
// KVQ_ERR_INVALID_ARG when the current CUDA device is not the cache's;
// otherwise *device = the cache's device.
kvq_status launch_device(const kvq_cache* c, int* device);

// ---------------------------------------------------------------------------
// launchers (defined in the kernel translation units)
// ---------------------------------------------------------------------------
cudaError_t launch_pt_update(int32_t* table, const PtUpdate& u, cudaStream_t s);

cudaError_t launch_append(const Layout& L, int layer, const Batch& b, int total_tokens,
                          const void* k, const void* v, cudaStream_t s);

cudaError_t launch_export(const Layout& L, int layer, int seq_id, int ring, int64_t tok0, int64_t n_tok,
                          void* k_codes, void* k_scales, void* v_codes, void* v_scales,
                          cudaStream_t s);

struct DecodePlan {
  int chunk_tokens;      // tokens per stage / work unit
  int n_items;           // n_seqs * n_kv_heads
  int64_t total_chunks;
  int64_t chunks_per_cta;
  int n_cta;             // CTAs launched (<= max_ctas)
  int max_ctas;          // CTA cap the workspace was sized for
};

// decode: workspace = partial slots [(max_ctas + n_items)][G][D + 2] fp32
size_t decode_workspace_bytes(int n_items, int max_ctas, int G, int D);
// Decode grids have at most one CTA per SM and never more than kMaxDecodeCtas (the
// in-kernel merge of a split item keeps one weight per CTA in shared memory).
constexpr int kMaxDecodeCtas = 256;
int decode_max_ctas(int num_sms);
int decode_chunk_tokens(const Layout& L, int G);
bool decode_tc_supported(const Layout& L, int G);
// k_new / v_new: fp16 [B, Hkv, D] rows of position len - 1 to quantise into the
// cache first (nullptr: plain decode); only when decode_fuses_append(L, G).
cudaError_t launch_decode(const Layout& L, int layer, const Batch& b, const DecodePlan& plan,
                          int n_q_heads, const void* q, void* out, const void* k_new, const void* v_new,
                          float scale_log2, void* workspace, cudaStream_t s);
bool decode_fuses_append(const Layout& L, int G);

// Two internal streams and events of a cache, on which chunked prefill alternates its waves.
struct PrefillStreams {
  cudaStream_t s[2];
  cudaEvent_t fork, join[2];
};
size_t prefill_workspace_bytes(const Layout& L, const Batch& b);
cudaError_t launch_prefill(const Layout& L, int layer, const Batch& b, int total_q, int n_q_heads,
                           const void* q, void* out, float scale, void* workspace, size_t ws_bytes,
                           const PrefillStreams& ps, cudaStream_t s);

}  // namespace kvq
