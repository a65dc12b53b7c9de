/*
 * kvq.h - C ABI of an asymmetric-precision quantized KV cache for NVIDIA B200 (sm_100a).
 *
 * What the library computes (source pages cited by title and section):
 *
 *  - "KVSplit - contexto 2 a 3 vezes mais longo em Apple Silicon"
 *    (pt.news.hada.io/topic?id=20969), sections "Problema que o KVSplit tenta
 *    resolver" and "Exemplos de uso e opcoes de CLI": keys and values of the
 *    attention KV cache are stored at independently chosen bit widths
 *    (--kvq-key / --kvq-val: 16, 8 or 4), e.g. K8V4 = 8-bit keys, 4-bit values.
 *  - Same page, "Uso de memoria conforme o comprimento da sequencia": the KV
 *    memory table is exact for 32-element blocks carrying one fp16 scale each
 *    (34 B per 8-bit block, 18 B per 4-bit block) with 256-token page
 *    capacity; kvq_cache_footprint / kvq_footprint_bytes reproduce it.
 *  - Same page, Hacker News reply on .gguf compatibility: the cache is quantised
 *    at run time as tokens are processed, independently of the weights
 *    (kvq_append).
 *  - Same page, "Exemplos de uso e opcoes de CLI" (--flash-attn): attention is
 *    read through the flash-attention path (kvq_decode_attn: split-KV
 *    flash-decoding; kvq_prefill_attn: causal chunk attention).
 *  - "Reutilizacao de Cache KV para Conversas Longas no Apple Silicon"
 *    (openclawradar.com), "Principais Descobertas e Benchmarks": keep the cache
 *    resident and process only the new tokens (append a chunk, then
 *    kvq_prefill_attn over cache + chunk).
 *
 * Storage format of one 32-element block along head_dim (the pages fix the
 * byte counts; the rounding rules are this library's reading, stated exactly):
 *    8-bit: d = fp16(fp32(amax / 127)); c_j = clamp(roundf(x_j / d), -127, 127)
 *           (fp32 division, ties away from zero; d == 0 gives c = 0); x^ = d * c.
 *    4-bit: m = element of largest |x| (lowest index on ties); d = fp16(m / -8);
 *           c_j = clamp(roundf(x_j / d), -8, 7); nibble u_j = c_j + 8;
 *           byte i (0..15) = u_i | u_{i+16} << 4; x^ = d * (u - 8).
 *   16-bit: fp16 copy.
 *
 * Conventions for every call:
 *  - Returns a kvq_status; never aborts or throws across the ABI.  Arguments
 *    are validated on the host before anything is launched; on a validation
 *    error nothing is modified.  Errors of earlier asynchronous work are
 *    reported by kvq_cache_check.
 *  - "device" pointers are CUDA global-memory addresses on the cache's device;
 *    "host" pointers are ordinary CPU memory read during the call only.  The
 *    caller owns every pointer it passes; the library owns the page pool,
 *    the page table and its host bookkeeping.
 *  - fp16 tensors are IEEE binary16, contiguous, row-major in the shapes given.
 *  - Work is enqueued on `stream` (NULL = legacy default stream).  Calls on one
 *    cache must be serialised by the caller (one host thread at a time, and
 *    device work ordered on one stream or by the caller's events).
 *  - Query head h reads KV head h / (n_q_heads / n_kv_heads).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t (a CUDA runtime / driver stream handle). */
typedef struct CUstream_st* kvq_stream_t;

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,    /* bad pointer, size, id, layer or shape          */
  KVQ_ERR_UNSUPPORTED = 2,    /* valid but not built (bit width, head_dim, ...) */
  KVQ_ERR_OUT_OF_MEMORY = 3,  /* device or host allocation failed               */
  KVQ_ERR_CAPACITY = 4,       /* page pool or per-sequence page table exhausted */
  KVQ_ERR_CUDA = 5,           /* a CUDA runtime call failed                     */
  KVQ_ERR_DEVICE_CHECK = 6,   /* a kernel gave up a bounded wait or found a bad index */
  KVQ_ERR_WORKSPACE = 7       /* workspace missing or smaller than required     */
} kvq_status;

/* Cache geometry.  k_bits / v_bits in {16, 8, 4}; head_dim in {64, 128};
 * page_tokens a multiple of 64 in [64, 4096] (0 selects 256); sequences are
 * named by ids 0 .. max_seqs-1; max_tokens is the pool capacity in tokens over
 * all sequences (rounded up to whole pages); max_seq_tokens (0 = max_tokens)
 * bounds one sequence's length and sizes its page-table row.
 * Per-layer precision (the "Layer-Specific Quantization" item of the KVSplit
 * page's "Configuracao recomendada e roadmap"): layer_k_bits / layer_v_bits,
 * when not NULL, are host arrays of n_layers bit widths that replace k_bits /
 * v_bits layer by layer (both or neither; read by kvq_cache_create and
 * kvq_footprint_bytes only, not kept).  Each layer is either fp16 for K and V
 * or quantized for both. */
typedef struct {
  int32_t n_layers;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t k_bits;
  int32_t v_bits;
  int32_t page_tokens;
  int32_t max_seqs;
  int32_t flags;            /* KVQ_CACHE_* bits */
  int64_t max_tokens;
  int64_t max_seq_tokens;
  const int32_t* layer_k_bits;   /* NULL or [n_layers] */
  const int32_t* layer_v_bits;   /* NULL or [n_layers] */
} kvq_cache_config;

/* flags: KVQ_CACHE_HOST_ONLY creates the page bookkeeping without touching a
 * GPU (no device memory); calls that would launch work then return
 * KVQ_ERR_UNSUPPORTED.  Used to test the host logic on machines without a GPU. */
#define KVQ_CACHE_HOST_ONLY 1
/* KVQ_CACHE_DECODE_TENSOR_CORES runs kvq_decode_attn on the tcgen05 tensor
 * cores where a kernel for the shape exists (8-bit keys, 4- or 8-bit values,
 * head_dim 128, 1 / 2 / 4 / 8 query heads per KV head): scores as int8 MMAs on
 * the stored key codes, PV as fp16 MMAs on values dequantised once per token.
 * Other shapes, and caches without the flag, use the CUDA-core kernel that
 * dequantises K and V in registers.  Results agree within the attention
 * tolerance; the flag only changes speed. */
#define KVQ_CACHE_DECODE_TENSOR_CORES 2

/* Most sequences one append / decode / prefill call may name. */
#define KVQ_MAX_BATCH 256

typedef struct kvq_cache kvq_cache;

/* Closed-form KV bytes of n_tokens of one sequence under cfg, over all layers:
 * *allocated_bytes counts whole pages (the pages' table), *used_bytes counts
 * the tokens only.  Pure host arithmetic; either output may be NULL. */
KVQ_API kvq_status kvq_footprint_bytes(const kvq_cache_config* cfg, int64_t n_tokens,
                               int64_t* allocated_bytes, int64_t* used_bytes);

/* Create a cache on the current CUDA device: one device allocation holding
 * every layer's pages (zero-filled), a device page table, and host
 * bookkeeping.  *out receives the handle (NULL on error). */
KVQ_API kvq_status kvq_cache_create(const kvq_cache_config* cfg, kvq_cache** out);

/* Free everything the cache owns.  Synchronises the device first.  NULL is a no-op. */
KVQ_API kvq_status kvq_cache_destroy(kvq_cache* cache);

/* Bytes of the whole pool, of the pages currently mapped to sequences, and of
 * the tokens held (all layers).  Any output may be NULL. */
KVQ_API kvq_status kvq_cache_footprint(const kvq_cache* cache, int64_t* pool_bytes,
                               int64_t* mapped_bytes, int64_t* used_bytes);

/* Grow sequences: for i < n_seqs, sequence seq_ids[i] gains n_new[i] >= 0
 * token positions at its end, mapping free pages as needed (host arrays).
 * Page-table updates are enqueued on `stream`.  The new positions hold no data
 * until kvq_append writes them, layer by layer.  All-or-nothing: on
 * KVQ_ERR_CAPACITY no sequence changes (the capacity check counts one page for
 * every shared partly filled last page it may have to copy).  A sequence id may
 * appear once. */
KVQ_API kvq_status kvq_seq_extend(kvq_cache* cache, int32_t n_seqs, const int32_t* seq_ids,
                          const int32_t* n_new, kvq_stream_t stream);

/* Drop a sequence: its length becomes 0 and each of its pages returns to the
 * pool unless another sequence still maps it (kvq_seq_fork). */
KVQ_API kvq_status kvq_seq_release(kvq_cache* cache, int32_t seq_id);

/* Shorten a sequence to new_len <= its length (rewind a chunk, or keep a
 * session's prefix and drop its last turn, as in reusing a conversation's
 * cache and processing only the new tokens: "Reutilizacao de Cache KV para
 * Conversas Longas no Apple Silicon", "Principais Descobertas e Benchmarks").
 * Whole pages past new_len are dropped (returned to the pool unless another
 * sequence still maps them).  Host bookkeeping only: the caller orders it after
 * device work that still reads the dropped positions. */
KVQ_API kvq_status kvq_seq_truncate(kvq_cache* cache, int32_t seq_id, int64_t new_len);

/* Share a prefix: empty sequence dst becomes the first n_tokens <= len(src)
 * positions of src, in every layer, by mapping the same physical pages
 * (reference-counted; no data is copied).  A page stays shared while neither
 * sequence writes into it; when kvq_seq_extend is about to add positions to a
 * partly filled page that another sequence still maps, it first copies that
 * page (all layers) to a private page on `stream` (copy-on-write), so appends
 * never change what the other sequence reads.  Release and truncate drop one
 * reference; a page returns to the pool with its last one.  This is the
 * keep-the-cache reuse of "Reutilizacao de Cache KV para Conversas Longas no
 * Apple Silicon" ("Principais Descobertas e Benchmarks") extended to several
 * conversations that start from one cached prefix.  Page-table updates are
 * enqueued on `stream`.  KVQ_ERR_INVALID_ARG if src == dst, dst is not empty or
 * n_tokens is outside [0, len(src)]. */
KVQ_API kvq_status kvq_seq_fork(kvq_cache* cache, int32_t src_seq, int32_t dst_seq, int64_t n_tokens,
                                kvq_stream_t stream);

/* Rotating window ("Reutilizacao de Cache KV para Conversas Longas no Apple
 * Silicon", "O Que Nao Funcionou": rotating the KV cache at 8192 tokens, which
 * gave the best tokens/s at the price of the earlier context).  Sequence seq_id,
 * which must be empty, keeps only its last window_tokens positions from now
 * on: its pages form a ring of window_tokens / page_tokens + 1 page-table slots,
 * so once the ring is full kvq_seq_extend reuses the page of the oldest
 * positions, which lie entirely before the window, and maps no new page.
 * kvq_decode_attn / kvq_decode_append_attn attend to positions
 * max(0, len - window_tokens) .. len - 1 (on the CUDA-core kernels).
 * window_tokens: 0 (no window, the default) or a positive multiple of
 * page_tokens with window_tokens / page_tokens + 1 <= the page-table row
 * (max_seq_tokens / page_tokens), else KVQ_ERR_INVALID_ARG / KVQ_ERR_CAPACITY.
 * A windowed sequence's length is bounded by 2^30 instead of max_seq_tokens;
 * one kvq_append may add at most window_tokens positions; kvq_export reads
 * positions inside the window only; kvq_seq_fork of or onto a windowed
 * sequence, kvq_seq_truncate after the ring wrapped and kvq_prefill_attn once
 * len > window_tokens return KVQ_ERR_UNSUPPORTED.  The window survives
 * kvq_seq_release. */
KVQ_API kvq_status kvq_seq_set_window(kvq_cache* cache, int32_t seq_id, int64_t window_tokens);

/* Current length (token positions) of a sequence. */
KVQ_API kvq_status kvq_seq_length(const kvq_cache* cache, int32_t seq_id, int64_t* len);

/* Physical page index of logical page `page` of a sequence (host bookkeeping;
 * -1 if unmapped).  For tests of the allocator. */
KVQ_API kvq_status kvq_seq_page(const kvq_cache* cache, int32_t seq_id, int32_t page, int32_t* phys);

/* Quantise-on-append.  For i < n_seqs (host arrays seq_ids, n_new), writes the
 * K and V of the LAST n_new[i] positions of sequence seq_ids[i] in `layer`,
 * i.e. positions [len - n_new[i], len).  k, v: device fp16
 * [sum_i n_new[i], n_kv_heads, head_dim], sequences' rows in call order.
 * Quantises every 32-element block along head_dim to the cache's K / V bit
 * widths (format above) and stores codes and scales into the sequence's pages.
 * k and v must be 16-byte aligned (KVQ_ERR_INVALID_ARG otherwise). */
KVQ_API kvq_status kvq_append(kvq_cache* cache, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                      const int32_t* n_new, const void* k, const void* v, kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn needs for a batch of n_seqs sequences with
 * n_q_heads query heads (independent of lengths).  Pure host arithmetic. */
KVQ_API kvq_status kvq_decode_workspace_size(const kvq_cache* cache, int32_t n_seqs, int32_t n_q_heads,
                                     size_t* bytes);

/* Decode attention, one query position per sequence: for i < n_seqs the query
 * q[i] (position len-1 of sequence seq_ids[i]) attends to cache positions
 * 0 .. len-1 of `layer`:  o = softmax(sigma * q K^T) V over the dequantised
 * K, V, sigma = softmax_scale (0 selects 1/sqrt(head_dim)).
 * q, out: device fp16 [n_seqs, n_q_heads, head_dim].  Split-KV flash-decoding:
 * partial (O, max, sum) per slice of the cache in `workspace` (device,
 * ws_bytes >= kvq_decode_workspace_size), merged by a log-sum-exp combine (for
 * quantized caches inside the same kernel, by the last CTA that finishes a
 * sequence's KV head; for fp16 caches and the tensor-core kernel, by a second
 * kernel).  The merge order is fixed, so results are deterministic.
 * Every named sequence must have len >= 1.  q, out and workspace must be
 * 16-byte aligned (KVQ_ERR_INVALID_ARG otherwise).
 * kvq_seq_extend, kvq_append, kvq_decode_attn and kvq_prefill_attn only
 * validate on the host and enqueue kernels on `stream` (no allocation, no
 * synchronisation), so a decode step made of them can be captured in a CUDA
 * graph and replayed. */
KVQ_API kvq_status kvq_decode_attn(kvq_cache* cache, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                           int32_t n_q_heads, const void* q, void* out, float softmax_scale,
                           void* workspace, size_t ws_bytes, kvq_stream_t stream);

/* One decode step of one layer: quantise-on-append of the token at position
 * len - 1 of every named sequence, then decode attention of its query over
 * positions 0 .. len - 1 (which include that token).  Same result as
 * kvq_append (n_new = 1 for each sequence) followed by kvq_decode_attn, in one
 * kernel launch for quantized caches (the CTA that streams the chunk holding
 * position len - 1 quantises the new row into the page just before copying
 * that chunk), two launches for fp16 caches and the tensor-core kernel.  The
 * positions must already exist (kvq_seq_extend), as for kvq_append.
 * k_new, v_new: device fp16 [n_seqs, n_kv_heads, head_dim], 16-byte aligned.
 * The KVSplit page quantises the cache at run time as tokens are processed
 * (Hacker News reply on .gguf files); the pages' small-model workloads
 * (22-layer table, "Principais resultados de benchmark") are one such step per
 * layer.  Other arguments, workspace and errors as kvq_decode_attn. */
KVQ_API kvq_status kvq_decode_append_attn(kvq_cache* cache, int32_t layer, int32_t n_seqs,
                                          const int32_t* seq_ids, int32_t n_q_heads, const void* q,
                                          const void* k_new, const void* v_new, void* out, float softmax_scale,
                                          void* workspace, size_t ws_bytes, kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn_layers needs for n_layers layers of a batch
 * of n_seqs sequences with n_q_heads query heads (independent of lengths and
 * of the layers' formats).  Pure host arithmetic. */
KVQ_API kvq_status kvq_decode_layers_workspace_size(const kvq_cache* cache, int32_t n_layers, int32_t n_seqs,
                                                    int32_t n_q_heads, size_t* bytes);

/* Layer-batched decode: the same result as calling, for l = 0 .. n_layers - 1,
 * kvq_decode_append_attn (k_new and v_new given) or kvq_decode_attn (both
 * NULL) on layer layer0 + l with that layer's rows of q, k_new, v_new and out,
 * but in one launch for every run of consecutive layers that share a format
 * and fit one batch (n_layers_in_run * n_seqs <= KVQ_MAX_BATCH): the kernel's
 * work list holds every (layer, sequence, KV head, slice) of the run, so its
 * CTAs stream the whole run's cache without a launch, a pipeline fill or a
 * tail per layer.  For use when every layer's query of the step is known at
 * once (a replayed or precomputed step); a model whose next layer's query
 * depends on this layer's output calls the per-layer functions.
 * Codes and scales written are identical to the per-layer calls'; the
 * attention outputs match them within rounding (the slices of an item may be
 * split among CTAs differently, which changes the fp32 summation order).
 * The step is the pages' small-model workload (KVSplit page, "Principais
 * resultados de benchmark": one decode step over every layer of a 22-layer
 * cache) with every layer's decode as in kvq_decode_attn.
 * q, out: device fp16 [n_layers, n_seqs, n_q_heads, head_dim];
 * k_new, v_new: device fp16 [n_layers, n_seqs, n_kv_heads, head_dim] or both
 * NULL; all 16-byte aligned.  workspace: device, ws_bytes >=
 * kvq_decode_layers_workspace_size (the runs reuse it in stream order).
 * Runs on the CUDA-core decode kernels (the tensor-core flag applies to the
 * per-layer calls only).  layer0 < 0, n_layers < 1 or layer0 + n_layers >
 * n_layers of the cache: KVQ_ERR_INVALID_ARG; other errors as
 * kvq_decode_append_attn. */
KVQ_API kvq_status kvq_decode_attn_layers(kvq_cache* cache, int32_t layer0, int32_t n_layers, int32_t n_seqs,
                                          const int32_t* seq_ids, int32_t n_q_heads, const void* q,
                                          const void* k_new, const void* v_new, void* out, float softmax_scale,
                                          void* workspace, size_t ws_bytes, kvq_stream_t stream);

/* Size of the scratch array compiled into the library for
 * kvq_decode_attn_noalloc (8 MiB per GPU that loads the library). */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/* kvq_decode_attn without a workspace argument: for callers that cannot
 * allocate device memory (a plugin inside a host application that owns all
 * GPU memory and passes only inputs and outputs, an engine whose allocator has
 * reserved the whole device, a serving loop that must never call cudaMalloc /
 * cudaFree because they can synchronise the device).  The source pages have no
 * counterpart of this call; it computes exactly what kvq_decode_attn computes.
 * The split-KV partials go to a fixed device array of KVQ_NOALLOC_SCRATCH_BYTES
 * inside the library instead of a caller buffer; the call allocates nothing.
 * The first call on each device looks up that array's device address
 * (cudaGetSymbolAddress, with the device current), so make it before any stream
 * capture.  All calls share the array and it keeps the last call's contents:
 * calls that overlap on the GPU race and must be ordered by the caller.
 * Returns KVQ_ERR_WORKSPACE when kvq_decode_workspace_size for this batch
 * exceeds KVQ_NOALLOC_SCRATCH_BYTES (nothing is launched then). */
KVQ_API kvq_status kvq_decode_attn_noalloc(kvq_cache* cache, int32_t layer, int32_t n_seqs,
                                           const int32_t* seq_ids, int32_t n_q_heads, const void* q,
                                           void* out, float softmax_scale, kvq_stream_t stream);

/* Workspace bytes kvq_prefill_attn needs for these sequences (host arrays;
 * uses their current lengths). */
KVQ_API kvq_status kvq_prefill_workspace_size(const kvq_cache* cache, int32_t n_seqs, const int32_t* seq_ids,
                                      const int32_t* q_lens, int32_t n_q_heads, size_t* bytes);

/* Chunked prefill attention.  For i < n_seqs, sequence seq_ids[i] has a chunk
 * of q_lens[i] >= 1 query rows at positions [len - q_lens[i], len) (already
 * appended to the cache); row r attends causally to positions
 * 0 .. len - q_lens[i] + r, i.e. the cached tokens and the chunk up to itself,
 * all dequantised.  q, out: device fp16 [sum_i q_lens[i], n_q_heads, head_dim].
 * Tensor cores (tcgen05) compute Q K^T and P V from fp16 operands with fp32
 * accumulation: the dequantised K enters as its fp16 rounding plus the
 * remainder (an e5m2 term against an e5m2 copy of q at head_dim 128, k to about
 * 2^-15; an fp16 term at head_dim 64, about 22 bits), V and P are rounded to fp16.
 * q, out and workspace must be 16-byte aligned. */
KVQ_API kvq_status kvq_prefill_attn(kvq_cache* cache, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                            const int32_t* q_lens, int32_t n_q_heads, const void* q, void* out,
                            float softmax_scale, void* workspace, size_t ws_bytes,
                            kvq_stream_t stream);

/* Content deduplication of full pages ("KVBoost acelera inferencia de LLMs em
 * 4,49x com cache reutilizavel", section "Contexto": cached chunks are found
 * again by a hash of their content).  Among the pages that every sequence
 * mapping them holds completely (all page_tokens positions below its length;
 * sequences with a rotating window excluded), pages whose bytes are identical in
 * every layer are merged: each page-table entry of a duplicate then names one
 * representative page, whose reference count grows by the duplicate's, and the
 * duplicate returns to the pool.  Candidates come from a 128-bit content hash
 * computed on the GPU and are merged only after a byte comparison, so different
 * contents are never merged.  Full pages are never written again (appends
 * write positions >= len; a truncate into a shared page leaves it to
 * copy-on-write), so reads are unchanged.  Synchronises `stream` (hash and
 * comparison results are read back); page-table updates are enqueued on it.
 * *pages_freed (may be NULL) receives the number of pages returned. */
KVQ_API kvq_status kvq_cache_dedup(kvq_cache* cache, kvq_stream_t stream, int64_t* pages_freed);

/* Copy tokens [tok0, tok0 + n_tok) of a sequence in `layer` out in canonical
 * form (device destinations, any may be NULL to skip):
 *   k_codes  int8 [n_tok, Hkv, D] (8-bit) | uint8 [n_tok, Hkv, D/2] (4-bit, packed
 *            as above) | fp16 [n_tok, Hkv, D] (16-bit); v_codes likewise;
 *   k_scales, v_scales fp16 [n_tok, Hkv, D/32] (ignored for 16-bit). */
KVQ_API kvq_status kvq_export(const kvq_cache* cache, int32_t layer, int32_t seq_id, int64_t tok0,
                      int64_t n_tok, void* k_codes, void* k_scales, void* v_codes, void* v_scales,
                      kvq_stream_t stream);

/* Synchronise `stream` and report errors of earlier work: KVQ_ERR_CUDA for a
 * failed launch or runtime error, KVQ_ERR_DEVICE_CHECK if a kernel recorded a
 * bounded-wait timeout or an out-of-range index (then *detail, if not NULL,
 * receives the recorded code).  Clears the recorded device code. */
KVQ_API kvq_status kvq_cache_check(kvq_cache* cache, kvq_stream_t stream, uint32_t* detail);

/* Static description of a status code. */
KVQ_API const char* kvq_status_string(kvq_status status);

/* Text of the last error on this thread (a CUDA error string or a validation
 * message); never NULL. */
KVQ_API const char* kvq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
