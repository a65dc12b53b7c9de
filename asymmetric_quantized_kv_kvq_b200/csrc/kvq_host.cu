// Host side of the C ABI declared in include/kvq.h: argument validation, the
// page allocator, page-table maintenance and kernel dispatch.  Every check
// runs before anything is enqueued; a failed check leaves the cache unchanged.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "kvq_internal.cuh"
#include "sm100_util.cuh"

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

kvq_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? KVQ_ERR_OUT_OF_MEMORY : KVQ_ERR_CUDA;
}

#define KVQ_CUDA(call, what)                    \
  do {                                          \
    cudaError_t e_ = (call);                    \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool bits_ok(int b) { return b == 4 || b == 8 || b == 16; }

// Supported (k_bits, v_bits) pairs: both fp16, or both quantised.
bool pair_supported(int kb, int vb) {
  if (kb == 16 || vb == 16) return kb == vb;
  return true;
}

int64_t bytes_per_token_head(int bits, int D) {
  if (bits == 16) return 2LL * D;
  if (bits == 8) return int64_t(D / 32) * 34;
  return int64_t(D / 32) * 18;
}

// Bit widths of one layer: the per-layer arrays when given, else the cache-wide pair.
int layer_k_bits(const kvq_cache_config* c, int layer) { return c->layer_k_bits ? c->layer_k_bits[layer] : c->k_bits; }
int layer_v_bits(const kvq_cache_config* c, int layer) { return c->layer_v_bits ? c->layer_v_bits[layer] : c->v_bits; }

kvq_status check_config(const kvq_cache_config* c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "config is NULL");
  if (c->n_layers < 1 || c->n_kv_heads < 1) return fail(KVQ_ERR_INVALID_ARG, "n_layers and n_kv_heads must be >= 1");
  if (c->n_layers > 4096) return fail(KVQ_ERR_INVALID_ARG, "n_layers must be <= 4096");
  if (c->head_dim <= 0 || c->head_dim % 32) return fail(KVQ_ERR_INVALID_ARG, "head_dim must be a positive multiple of 32");
  if (!c->layer_k_bits != !c->layer_v_bits)
    return fail(KVQ_ERR_INVALID_ARG, "layer_k_bits and layer_v_bits must both be given or both be NULL");
  for (int l = 0; l < c->n_layers; ++l) {
    const int kb = layer_k_bits(c, l), vb = layer_v_bits(c, l);
    if (!bits_ok(kb) || !bits_ok(vb)) return fail(KVQ_ERR_INVALID_ARG, "layer %d: k_bits and v_bits must be 16, 8 or 4", l);
    if (!pair_supported(kb, vb)) return fail(KVQ_ERR_UNSUPPORTED, "layer %d: K%dV%d not built", l, kb, vb);
    if (!c->layer_k_bits) break;
  }
  if (c->head_dim != 64 && c->head_dim != 128) return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d not built (64, 128)", c->head_dim);
  int P = c->page_tokens ? c->page_tokens : 256;
  if (P < 64 || P > 4096 || P % 64) return fail(KVQ_ERR_INVALID_ARG, "page_tokens must be a multiple of 64 in [64, 4096]");
  if (c->max_seqs < 1 || c->max_seqs > (1 << 22)) return fail(KVQ_ERR_INVALID_ARG, "max_seqs out of range");
  if (c->max_tokens < 1) return fail(KVQ_ERR_INVALID_ARG, "max_tokens must be >= 1");
  int64_t mst = c->max_seq_tokens ? c->max_seq_tokens : c->max_tokens;
  if (mst < 1 || mst > (int64_t(1) << 30)) return fail(KVQ_ERR_INVALID_ARG, "max_seq_tokens out of range (<= 2^30)");
  if (c->flags & ~(KVQ_CACHE_HOST_ONLY | KVQ_CACHE_DECODE_TENSOR_CORES)) return fail(KVQ_ERR_INVALID_ARG, "unknown flags");
  int64_t pages = (c->max_tokens + P - 1) / P;
  if (pages > (int64_t(1) << 30)) return fail(KVQ_ERR_INVALID_ARG, "max_tokens too large");
  int64_t mpps = (mst + P - 1) / P;
  if (int64_t(c->max_seqs) * mpps > (int64_t(1) << 31) - 1) return fail(KVQ_ERR_INVALID_ARG, "page table too large");
  return KVQ_OK;
}

}  // namespace

kvq_status kvq::set_last_error(kvq_status s, const char* msg) {
  g_last_error = msg;
  return s;
}

struct kvq_cache {
  kvq_cache_config cfg{};
  bool host_only = false;
  int device = 0;
  int num_sms = 148;
  kvq::Layout L{};                   // cache-wide fields (pool = start of layer 0)
  std::vector<kvq::Layout> layers;   // per-layer views: pool = the layer's region, that layer's bits
  std::vector<int32_t> k_bits, v_bits;
  int64_t pool_bytes = 0;
  int64_t bytes_per_token = 0;       // all layers, K + V codes and scales
  int64_t bytes_per_page = 0;        // all layers, all heads
  int32_t* d_page_table = nullptr;
  uint32_t* d_err = nullptr;
  int32_t* d_counters = nullptr;     // decode split-item counters, [KVQ_MAX_BATCH * n_kv_heads]
  uint32_t* d_dedup = nullptr;       // page hashes [kDedupBatch][4] + compare flags [kDedupBatch]
  kvq::PrefillStreams pstreams{};    // internal streams / events of chunked prefill's waves
  std::vector<int32_t> table;        // host mirror of the page table
  std::vector<int64_t> len;          // tokens per sequence
  std::vector<int32_t> mapped;       // pages mapped per sequence
  std::vector<int32_t> free_pages;   // stack; back() is handed out next
  std::vector<int32_t> refs;         // sequences mapping each physical page (0 = free)
  std::vector<int64_t> window;       // rotating-window length per sequence (0 = keep every token)
  int64_t mapped_pages = 0;          // physical pages in use (each counted once)
};

namespace {

void destroy_streams(kvq_cache* c) {
  for (int k = 0; k < 2; ++k) {
    if (c->pstreams.s[k]) cudaStreamDestroy(c->pstreams.s[k]);
    if (c->pstreams.join[k]) cudaEventDestroy(c->pstreams.join[k]);
  }
  if (c->pstreams.fork) cudaEventDestroy(c->pstreams.fork);
  c->pstreams = kvq::PrefillStreams{};
}

kvq_status check_cache(const kvq_cache* c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
  return KVQ_OK;
}

kvq_status check_seq(const kvq_cache* c, int32_t id) {
  if (id < 0 || id >= c->cfg.max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id %d out of range", id);
  return KVQ_OK;
}

kvq_status check_ids(const kvq_cache* c, int32_t n, const int32_t* ids) {
  if (n < 1 || n > kvq::kMaxBatch) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [1, %d]", kvq::kMaxBatch);
  if (!ids) return fail(KVQ_ERR_INVALID_ARG, "seq_ids is NULL");
  std::vector<int32_t> sorted(ids, ids + n);
  for (int i = 0; i < n; ++i)
    if (kvq_status s = check_seq(c, ids[i])) return s;
  std::sort(sorted.begin(), sorted.end());
  for (int i = 1; i < n; ++i)
    if (sorted[i] == sorted[i - 1]) return fail(KVQ_ERR_INVALID_ARG, "sequence id %d repeated", sorted[i]);
  return KVQ_OK;
}

kvq_status check_layer(const kvq_cache* c, int32_t layer) {
  if (layer < 0 || layer >= c->cfg.n_layers) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  return KVQ_OK;
}

// Rotating window: a sequence with a window of W tokens keeps its pages in a ring
// of W / page_tokens + 1 page-table slots (logical page p in slot p % ring), which
// always holds the last W positions; 0 for a linear page table.
int32_t ring_pages(const kvq_cache* c, int32_t id) {
  return c->window[id] ? int32_t(c->window[id] / c->L.page_tokens + 1) : 0;
}
size_t slot_index(const kvq_cache* c, int32_t id, int64_t page) {
  return size_t(id) * c->L.max_pages_per_seq + size_t(kvq::page_slot(int(page), ring_pages(c, id)));
}
// Slots a sequence of nl positions maps.
int32_t slots_for(const kvq_cache* c, int32_t id, int64_t nl) {
  const int P = c->L.page_tokens;
  const int64_t pages = (nl + P - 1) / P;
  const int32_t R = ring_pages(c, id);
  return int32_t(R && pages > R ? R : pages);
}
// First position attended by a query at the sequence's end.
int64_t first_attended(const kvq_cache* c, int32_t id) {
  const int64_t w = c->window[id], n = c->len[id];
  return w && n > w ? n - w : 0;
}
// True once a windowed sequence has reused a ring slot (its logical pages no longer equal its slots).
bool wrapped(const kvq_cache* c, int32_t id) {
  const int32_t R = ring_pages(c, id);
  const int P = c->L.page_tokens;
  return R && (c->len[id] + P - 1) / P > R;
}

// Host-side fault injection for tests: with KVQ_INJECT_PT_FAILURE=k (k >= 1) in
// the environment, the k-th page-table enqueue of every kvq_seq_extend /
// kvq_seq_fork call fails as if the launch had failed (also for host-only
// caches, which enqueue nothing), so the rollback below runs on the CPU.
bool injected_pt_failure(int nth) {
  const char* f = std::getenv("KVQ_INJECT_PT_FAILURE");
  return f && std::atoi(f) == nth;
}

// Undo log of one kvq_seq_extend / kvq_seq_fork.  Those calls change the host
// bookkeeping as they go and enqueue page copies and page-table updates; if an
// enqueue fails part way, every change is put back in reverse order (and the
// page-table entries already enqueued are restored on the stream, best effort),
// so the call is all-or-nothing for the caller.
struct Journal {
  enum Kind : int32_t { kTake, kDrop, kRef, kSlot, kLen, kMapped };
  struct Op {
    Kind kind;
    int32_t a;     // page, table slot or sequence id
    int64_t old;   // previous value (slot entry, length, mapped pages)
  };
  std::vector<Op> ops;
  void add(Kind k, int32_t a, int64_t old = 0) { ops.push_back({k, a, old}); }
};

// Physical page bookkeeping: a page leaves the free stack with one reference,
// gains one per sequence that shares it (kvq_seq_fork) and returns to the stack
// when its last reference is dropped.
int32_t take_page(kvq_cache* c, Journal* j = nullptr) {
  const int32_t page = c->free_pages.back();
  c->free_pages.pop_back();
  c->refs[page] = 1;
  c->mapped_pages++;
  if (j) j->add(Journal::kTake, page);
  return page;
}
void drop_page(kvq_cache* c, int32_t page, Journal* j = nullptr) {
  if (--c->refs[page] == 0) {
    c->free_pages.push_back(page);
    c->mapped_pages--;
  }
  if (j) j->add(Journal::kDrop, page);
}
void set_slot(kvq_cache* c, size_t slot, int32_t val, Journal* j) {
  j->add(Journal::kSlot, int32_t(slot), c->table[slot]);
  c->table[slot] = val;
}

// Puts the host bookkeeping back as it was before the journal's first change.
void undo(kvq_cache* c, const Journal& j) {
  for (auto it = j.ops.rbegin(); it != j.ops.rend(); ++it) {
    switch (it->kind) {
      case Journal::kTake:            // the page was popped from the free stack with one reference
        c->refs[it->a] = 0;
        c->mapped_pages--;
        c->free_pages.push_back(it->a);
        break;
      case Journal::kDrop:            // a reference was dropped; the last one pushed the page back
        if (c->refs[it->a] == 0) {
          c->free_pages.pop_back();
          c->mapped_pages++;
        }
        c->refs[it->a]++;
        break;
      case Journal::kRef: c->refs[it->a]--; break;
      case Journal::kSlot: c->table[size_t(it->a)] = int32_t(it->old); break;
      case Journal::kLen: c->len[it->a] = it->old; break;
      case Journal::kMapped: c->mapped[it->a] = int32_t(it->old); break;
    }
  }
}

// Undo after a failed enqueue: the host bookkeeping goes back, and the
// page-table entries of the first `flushed` journal entries, already enqueued,
// are set back to their old values on the stream (best effort: the enqueue
// that failed may fail again, which kvq_cache_check then reports).
void rollback(kvq_cache* c, const Journal& j, size_t flushed, kvq_stream_t stream) {
  if (!c->host_only && flushed) {
    kvq::PtUpdate upd;
    upd.n = 0;
    for (size_t i = flushed; i-- > 0;) {
      const Journal::Op& op = j.ops[i];
      if (op.kind != Journal::kSlot) continue;
      upd.idx[upd.n] = op.a;
      upd.val[upd.n] = int32_t(op.old);
      if (++upd.n == kvq::kMaxPtUpdates) {
        (void)kvq::launch_pt_update(c->d_page_table, upd, (cudaStream_t)stream);
        upd.n = 0;
      }
    }
    (void)kvq::launch_pt_update(c->d_page_table, upd, (cudaStream_t)stream);
  }
  undo(c, j);
}

// Work is enqueued on the caller's stream with the caller's current device:
// that device must be the one the cache lives on.
kvq_status same_device(const kvq_cache* c) {
  if (c->host_only) return KVQ_OK;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVQ_ERR_CUDA, "cudaGetDevice failed");
  if (dev != c->device)
    return fail(KVQ_ERR_INVALID_ARG, "the current CUDA device is %d but the cache lives on device %d", dev, c->device);
  return KVQ_OK;
}

kvq_status need_device(const kvq_cache* c) {
  if (c->host_only) return fail(KVQ_ERR_UNSUPPORTED, "cache was created host-only");
  return same_device(c);
}

}  // namespace

kvq_status kvq::launch_device(const kvq_cache* c, int* device) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = need_device(c)) return s;
  *device = c->device;
  return KVQ_OK;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

kvq_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  return KVQ_OK;
}

}  // namespace

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported";
    case KVQ_ERR_OUT_OF_MEMORY: return "out of memory";
    case KVQ_ERR_CAPACITY: return "page capacity exhausted";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_DEVICE_CHECK: return "device-side check failed";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* kvq_last_error(void) { return g_last_error.c_str(); }

kvq_status kvq_footprint_bytes(const kvq_cache_config* cfg, int64_t n_tokens, int64_t* allocated, int64_t* used) {
  if (kvq_status s = check_config(cfg)) return s;
  if (n_tokens < 0) return fail(KVQ_ERR_INVALID_ARG, "n_tokens must be >= 0");
  int P = cfg->page_tokens ? cfg->page_tokens : 256;
  int64_t per = 0;   // bytes of one token over all layers
  for (int l = 0; l < cfg->n_layers; ++l)
    per += int64_t(cfg->n_kv_heads) * (bytes_per_token_head(layer_k_bits(cfg, l), cfg->head_dim) +
                                       bytes_per_token_head(layer_v_bits(cfg, l), cfg->head_dim));
  int64_t pages = (n_tokens + P - 1) / P;
  if (allocated) *allocated = pages * P * per;
  if (used) *used = n_tokens * per;
  return KVQ_OK;
}

kvq_status kvq_cache_create(const kvq_cache_config* cfg, kvq_cache** out) {
  if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (kvq_status s = check_config(cfg)) return s;
  kvq_cache* c = new (std::nothrow) kvq_cache();
  if (!c) return fail(KVQ_ERR_OUT_OF_MEMORY, "host allocation failed");
  c->cfg = *cfg;
  if (!c->cfg.page_tokens) c->cfg.page_tokens = 256;
  if (!c->cfg.max_seq_tokens) c->cfg.max_seq_tokens = c->cfg.max_tokens;
  c->host_only = (cfg->flags & KVQ_CACHE_HOST_ONLY) != 0;

  const int P = c->cfg.page_tokens, D = c->cfg.head_dim, H = c->cfg.n_kv_heads;
  kvq::Layout& L = c->L;
  L.n_kv_heads = H;
  L.n_layers = c->cfg.n_layers;
  L.decode_tc = (cfg->flags & KVQ_CACHE_DECODE_TENSOR_CORES) ? 1 : 0;
  // Device-side fault injection for tests: with KVQ_TEST_WITHHOLD_ARRIVAL=1 in the
  // environment when the cache is created, the quantized decode kernel's CTA 0
  // never fills its first stage and every wait of the kernel gives up after
  // 1 ms instead of 2 s, so the bounded wait runs out, the kernel records
  // kErrWaitTimeout and returns, and kvq_cache_check reports it.  No wait is
  // unbounded, so nothing hangs.
  if (const char* f = std::getenv("KVQ_TEST_WITHHOLD_ARRIVAL"); f && f[0] == '1') {
    L.test_withhold = 1;
    L.wait_ns = 1000000ull;
  } else {
    L.test_withhold = 0;
    L.wait_ns = kvq::kWaitLimitNs;
  }
  L.page_tokens = P;
  L.head_dim = D;
  L.s_row = (D / kvq::QK) * 2;
  L.n_pages = int32_t((c->cfg.max_tokens + P - 1) / P);
  L.max_pages_per_seq = int32_t((c->cfg.max_seq_tokens + P - 1) / P);

  try {
    // per-layer views of the pool: pool[layer] is n_pages * H head blocks of that layer's format
    // (the per-layer bit widths of the KVSplit page's roadmap, "Configuracao recomendada e roadmap")
    c->layers.assign(c->cfg.n_layers, L);
    c->k_bits.resize(c->cfg.n_layers);
    c->v_bits.resize(c->cfg.n_layers);
    for (int l = 0; l < c->cfg.n_layers; ++l) {
      kvq::Layout& V = c->layers[l];
      c->k_bits[l] = V.k_bits = layer_k_bits(cfg, l);
      c->v_bits[l] = V.v_bits = layer_v_bits(cfg, l);
      V.k_row = kvq::code_row_bytes(V.k_bits, D);
      V.v_row = kvq::code_row_bytes(V.v_bits, D);
      const int ks = V.k_bits == 16 ? 0 : V.s_row, vs = V.v_bits == 16 ? 0 : V.s_row;
      V.k_scales_off = P * V.k_row;
      V.v_codes_off = V.k_scales_off + P * ks;
      V.v_scales_off = V.v_codes_off + P * V.v_row;
      V.head_block = int64_t(V.v_scales_off) + int64_t(P) * vs;
      V.n_layers = 1;
      c->bytes_per_token += int64_t(H) * (V.k_row + ks + V.v_row + vs);
      c->bytes_per_page += int64_t(H) * V.head_block;
    }
    c->cfg.layer_k_bits = nullptr;   // the caller's arrays are not kept
    c->cfg.layer_v_bits = nullptr;
    L.k_bits = c->k_bits[0];
    L.v_bits = c->v_bits[0];
    c->pool_bytes = int64_t(L.n_pages) * c->bytes_per_page;

    // host-side fault injection for tests: the environment variable
    // KVQ_INJECT_ALLOC_FAILURE=1 makes this allocation fail, through the same
    // cleanup as a real one
    if (const char* f = std::getenv("KVQ_INJECT_ALLOC_FAILURE"); f && f[0] == '1') throw std::bad_alloc();
    c->table.assign(size_t(c->cfg.max_seqs) * L.max_pages_per_seq, -1);
    c->len.assign(c->cfg.max_seqs, 0);
    c->mapped.assign(c->cfg.max_seqs, 0);
    c->free_pages.resize(L.n_pages);
    c->refs.assign(L.n_pages, 0);
    c->window.assign(c->cfg.max_seqs, 0);
  } catch (...) {
    delete c;
    return fail(KVQ_ERR_OUT_OF_MEMORY, "host bookkeeping allocation failed");
  }
  for (int32_t i = 0; i < L.n_pages; ++i) c->free_pages[i] = L.n_pages - 1 - i;  // page 0 first

  if (!c->host_only) {
    cudaError_t e;
    if ((e = cudaGetDevice(&c->device)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device)) != cudaSuccess) {
      delete c;
      return cuda_fail(e, "cudaGetDevice");
    }
    auto cleanup = [&](cudaError_t err, const char* what) {
      if (L.pool) cudaFree(L.pool);
      if (c->d_page_table) cudaFree(c->d_page_table);
      if (c->d_err) cudaFree(c->d_err);
      if (c->d_counters) cudaFree(c->d_counters);
      if (c->d_dedup) cudaFree(c->d_dedup);
      destroy_streams(c);
      delete c;
      return cuda_fail(err, what);
    };
    const size_t counter_bytes = size_t(kvq::kMaxBatch) * H * sizeof(int32_t);
    if ((e = cudaMalloc(&L.pool, size_t(c->pool_bytes))) != cudaSuccess) return cleanup(e, "cudaMalloc(page pool)");
    if ((e = cudaMalloc(&c->d_page_table, c->table.size() * sizeof(int32_t))) != cudaSuccess)
      return cleanup(e, "cudaMalloc(page table)");
    if ((e = cudaMalloc(&c->d_err, sizeof(uint32_t))) != cudaSuccess) return cleanup(e, "cudaMalloc(error word)");
    if ((e = cudaMemset(L.pool, 0, size_t(c->pool_bytes))) != cudaSuccess) return cleanup(e, "cudaMemset(pool)");
    if ((e = cudaMemset(c->d_page_table, 0xFF, c->table.size() * sizeof(int32_t))) != cudaSuccess)
      return cleanup(e, "cudaMemset(page table)");
    if ((e = cudaMemset(c->d_err, 0, sizeof(uint32_t))) != cudaSuccess) return cleanup(e, "cudaMemset(err)");
    if ((e = cudaMalloc(&c->d_counters, counter_bytes)) != cudaSuccess) return cleanup(e, "cudaMalloc(counters)");
    if ((e = cudaMemset(c->d_counters, 0, counter_bytes)) != cudaSuccess) return cleanup(e, "cudaMemset(counters)");
    if ((e = cudaMalloc(&c->d_dedup, size_t(kvq::kDedupBatch) * 5 * sizeof(uint32_t))) != cudaSuccess)
      return cleanup(e, "cudaMalloc(dedup)");
    for (int k = 0; k < 2; ++k)
      if ((e = cudaStreamCreateWithFlags(&c->pstreams.s[k], cudaStreamNonBlocking)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&c->pstreams.join[k], cudaEventDisableTiming)) != cudaSuccess)
        return cleanup(e, "prefill streams");
    if ((e = cudaEventCreateWithFlags(&c->pstreams.fork, cudaEventDisableTiming)) != cudaSuccess)
      return cleanup(e, "prefill streams");
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cleanup(e, "cudaDeviceSynchronize");
    L.page_table = c->d_page_table;
    L.err = c->d_err;
    L.counters = c->d_counters;
    int64_t base = 0;
    for (kvq::Layout& V : c->layers) {
      V.pool = L.pool + base;
      V.page_table = L.page_table;
      V.err = L.err;
      V.counters = L.counters;
      base += int64_t(L.n_pages) * H * V.head_block;
    }
  }
  *out = c;
  return KVQ_OK;
}

kvq_status kvq_cache_destroy(kvq_cache* c) {
  if (!c) return KVQ_OK;
  kvq_status st = KVQ_OK;
  if (!c->host_only) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) st = cuda_fail(e, "cudaDeviceSynchronize");
    cudaFree(c->L.pool);
    cudaFree(c->d_page_table);
    cudaFree(c->d_err);
    cudaFree(c->d_counters);
    cudaFree(c->d_dedup);
    destroy_streams(c);
  }
  delete c;
  return st;
}

kvq_status kvq_cache_footprint(const kvq_cache* c, int64_t* pool, int64_t* mapped, int64_t* used) {
  if (kvq_status s = check_cache(c)) return s;
  if (pool) *pool = c->pool_bytes;
  if (mapped) *mapped = c->mapped_pages * c->bytes_per_page;
  if (used) {
    int64_t t = 0;
    for (int64_t x : c->len) t += x;
    *used = t * c->bytes_per_token;
  }
  return KVQ_OK;
}

kvq_status kvq_seq_set_window(kvq_cache* c, int32_t id, int64_t window_tokens) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_seq(c, id)) return s;
  if (c->len[id] != 0 || c->mapped[id] != 0) return fail(KVQ_ERR_INVALID_ARG, "sequence %d is not empty", id);
  const int P = c->L.page_tokens;
  if (window_tokens < 0 || window_tokens % P)
    return fail(KVQ_ERR_INVALID_ARG, "window must be 0 or a positive multiple of page_tokens (%d)", P);
  if (window_tokens / P + 1 > c->L.max_pages_per_seq)
    return fail(KVQ_ERR_CAPACITY, "a window of %lld tokens needs %lld page-table slots > %d", (long long)window_tokens,
                (long long)(window_tokens / P + 1), c->L.max_pages_per_seq);
  c->window[id] = window_tokens;
  return KVQ_OK;
}

kvq_status kvq_seq_length(const kvq_cache* c, int32_t id, int64_t* len) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_seq(c, id)) return s;
  if (!len) return fail(KVQ_ERR_INVALID_ARG, "len is NULL");
  *len = c->len[id];
  return KVQ_OK;
}

kvq_status kvq_seq_page(const kvq_cache* c, int32_t id, int32_t page, int32_t* phys) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_seq(c, id)) return s;
  if (!phys) return fail(KVQ_ERR_INVALID_ARG, "phys is NULL");
  if (page < 0 || page >= c->L.max_pages_per_seq) return fail(KVQ_ERR_INVALID_ARG, "page index out of range");
  *phys = c->table[size_t(id) * c->L.max_pages_per_seq + page];
  return KVQ_OK;
}

kvq_status kvq_seq_extend(kvq_cache* c, int32_t n, const int32_t* ids, const int32_t* n_new, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_ids(c, n, ids)) return s;
  if (!n_new) return fail(KVQ_ERR_INVALID_ARG, "n_new is NULL");
  if (kvq_status s = same_device(c)) return s;
  const int P = c->L.page_tokens;
  // a sequence whose last page is partly filled and shared with another sequence
  // (kvq_seq_fork) gets a private copy of that page before new tokens land in it
  auto shared_tail = [&](int32_t id) -> int32_t {
    if (c->len[id] % P == 0) return -1;
    const int32_t p = int32_t(c->len[id] / P);
    return c->refs[c->table[slot_index(c, id, p)]] > 1 ? p : -1;
  };
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    if (n_new[i] < 0) return fail(KVQ_ERR_INVALID_ARG, "n_new[%d] < 0", i);
    int64_t nl = c->len[ids[i]] + n_new[i];
    // a rotating window reuses its ring of pages: only its positions are bounded (kernels index in int32)
    const int64_t limit = c->window[ids[i]] ? (int64_t(1) << 30) : c->cfg.max_seq_tokens;
    if (nl > limit)
      return fail(KVQ_ERR_CAPACITY, "sequence %d would hold %lld tokens > %lld", ids[i], (long long)nl,
                  (long long)limit);
    need += slots_for(c, ids[i], nl) - c->mapped[ids[i]];
    if (n_new[i] > 0 && shared_tail(ids[i]) >= 0) ++need;
  }
  if (need > int64_t(c->free_pages.size()))
    return fail(KVQ_ERR_CAPACITY, "need %lld pages, %zu free", (long long)need, c->free_pages.size());

  Journal j;
  kvq::PtUpdate upd;
  upd.n = 0;
  size_t flushed = 0;   // journal entries whose page-table updates were enqueued
  int n_flush = 0;
  auto flush = [&]() -> kvq_status {
    if (upd.n == 0) return KVQ_OK;
    if (injected_pt_failure(++n_flush)) {
      upd.n = 0;
      return fail(KVQ_ERR_CUDA, "page-table update: injected failure (KVQ_INJECT_PT_FAILURE)");
    }
    if (c->host_only) { upd.n = 0; flushed = j.ops.size(); return KVQ_OK; }
    const cudaError_t e = kvq::launch_pt_update(c->d_page_table, upd, (cudaStream_t)stream);
    upd.n = 0;
    if (e == cudaSuccess) flushed = j.ops.size();
    return launched(e, "page-table update");
  };
  auto queue = [&](size_t slot, int32_t page) -> kvq_status {
    set_slot(c, slot, page, &j);
    upd.idx[upd.n] = int32_t(slot);
    upd.val[upd.n] = page;
    return ++upd.n == kvq::kMaxPtUpdates ? flush() : KVQ_OK;
  };
  kvq_status st = KVQ_OK;
  for (int i = 0; i < n && st == KVQ_OK; ++i) {
    const int32_t id = ids[i];
    const int64_t nl = c->len[id] + n_new[i];
    const int32_t want = slots_for(c, id, nl);
    const int32_t tail = n_new[i] > 0 ? shared_tail(id) : -1;
    if (tail >= 0) {
      const size_t slot = slot_index(c, id, tail);
      const int32_t from = c->table[slot], to = take_page(c, &j);
      if (!c->host_only) {
        // the page's head blocks of one layer are contiguous: one copy per layer
        for (int32_t layer = 0; layer < c->cfg.n_layers && st == KVQ_OK; ++layer) {
          const kvq::Layout& V = c->layers[layer];
          const int64_t bytes = int64_t(V.n_kv_heads) * V.head_block;
          const cudaError_t e = cudaMemcpyAsync(V.head_ptr(0, to, 0), V.head_ptr(0, from, 0), size_t(bytes),
                                                cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
          if (e != cudaSuccess) st = cuda_fail(e, "copy of a shared page");
        }
        if (st != KVQ_OK) break;
      }
      drop_page(c, from, &j);
      st = queue(slot, to);
    }
    // new slots (a ring's slots are only ever added until the ring is full; after that the
    // slot of the oldest page, entirely before the window, is written again)
    while (st == KVQ_OK && c->mapped[id] < want) {
      const int32_t page = take_page(c, &j);
      const size_t slot = size_t(id) * c->L.max_pages_per_seq + c->mapped[id];
      j.add(Journal::kMapped, id, c->mapped[id]);
      c->mapped[id]++;
      st = queue(slot, page);
    }
    if (st == KVQ_OK) {
      j.add(Journal::kLen, id, c->len[id]);
      c->len[id] = nl;
    }
  }
  if (st == KVQ_OK) st = flush();
  if (st != KVQ_OK) rollback(c, j, flushed, stream);
  return st;
}

kvq_status kvq_seq_release(kvq_cache* c, int32_t id) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_seq(c, id)) return s;
  for (int32_t p = c->mapped[id] - 1; p >= 0; --p) {
    int32_t& slot = c->table[size_t(id) * c->L.max_pages_per_seq + p];
    drop_page(c, slot);
    slot = -1;
  }
  c->mapped[id] = 0;
  c->len[id] = 0;
  return KVQ_OK;
}

kvq_status kvq_seq_truncate(kvq_cache* c, int32_t id, int64_t new_len) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_seq(c, id)) return s;
  if (new_len < 0 || new_len > c->len[id])
    return fail(KVQ_ERR_INVALID_ARG, "new_len %lld outside [0, len = %lld]", (long long)new_len, (long long)c->len[id]);
  if (wrapped(c, id) && new_len != c->len[id])
    return fail(KVQ_ERR_UNSUPPORTED, "sequence %d: truncate after its rotating window wrapped", id);
  const int P = c->L.page_tokens;
  const int32_t keep = int32_t((new_len + P - 1) / P);
  for (int32_t p = c->mapped[id] - 1; p >= keep; --p) {
    int32_t& slot = c->table[size_t(id) * c->L.max_pages_per_seq + p];
    drop_page(c, slot);
    slot = -1;
  }
  c->mapped[id] = keep;
  c->len[id] = new_len;
  return KVQ_OK;
}

kvq_status kvq_seq_fork(kvq_cache* c, int32_t src, int32_t dst, int64_t n_tokens, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_seq(c, src)) return s;
  if (kvq_status s = check_seq(c, dst)) return s;
  if (src == dst) return fail(KVQ_ERR_INVALID_ARG, "fork of sequence %d onto itself", src);
  if (c->window[src] || c->window[dst]) return fail(KVQ_ERR_UNSUPPORTED, "fork of a rotating-window sequence");
  if (c->len[dst] != 0 || c->mapped[dst] != 0) return fail(KVQ_ERR_INVALID_ARG, "sequence %d is not empty", dst);
  if (n_tokens < 0 || n_tokens > c->len[src])
    return fail(KVQ_ERR_INVALID_ARG, "n_tokens %lld outside [0, len = %lld]", (long long)n_tokens,
                (long long)c->len[src]);
  if (kvq_status s = same_device(c)) return s;
  const int P = c->L.page_tokens;
  const int32_t pages = int32_t((n_tokens + P - 1) / P);
  Journal j;
  kvq::PtUpdate upd;
  upd.n = 0;
  size_t flushed = 0;
  int n_flush = 0;
  kvq_status st = KVQ_OK;
  for (int32_t p = 0; p < pages && st == KVQ_OK; ++p) {
    const int32_t page = c->table[size_t(src) * c->L.max_pages_per_seq + p];
    const size_t slot = size_t(dst) * c->L.max_pages_per_seq + p;
    set_slot(c, slot, page, &j);
    c->refs[page]++;
    j.add(Journal::kRef, page);
    upd.idx[upd.n] = int32_t(slot);
    upd.val[upd.n] = page;
    if (++upd.n == kvq::kMaxPtUpdates || p == pages - 1) {
      if (injected_pt_failure(++n_flush))
        st = fail(KVQ_ERR_CUDA, "page-table update: injected failure (KVQ_INJECT_PT_FAILURE)");
      else if (!c->host_only)
        st = launched(kvq::launch_pt_update(c->d_page_table, upd, (cudaStream_t)stream), "page-table update");
      if (st == KVQ_OK) flushed = j.ops.size();
      upd.n = 0;
    }
  }
  if (st != KVQ_OK) {
    rollback(c, j, flushed, stream);
    return st;
  }
  c->mapped[dst] = pages;
  c->len[dst] = n_tokens;
  return KVQ_OK;
}

kvq_status kvq_append(kvq_cache* c, int32_t layer, int32_t n, const int32_t* ids, const int32_t* n_new,
                      const void* k, const void* v, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_layer(c, layer)) return s;
  if (kvq_status s = check_ids(c, n, ids)) return s;
  if (!n_new) return fail(KVQ_ERR_INVALID_ARG, "n_new is NULL");
  kvq::Batch b;
  b.n = n;
  int64_t total = 0;
  for (int i = 0; i < n; ++i) {
    if (n_new[i] < 0 || n_new[i] > c->len[ids[i]])
      return fail(KVQ_ERR_INVALID_ARG, "n_new[%d] = %d outside [0, len = %lld]", i, n_new[i], (long long)c->len[ids[i]]);
    if (c->window[ids[i]] && n_new[i] > c->window[ids[i]])
      return fail(KVQ_ERR_INVALID_ARG, "n_new[%d] = %d exceeds the sequence's window", i, n_new[i]);
    b.s[i] = {ids[i], int32_t(c->len[ids[i]] - n_new[i]), n_new[i], int32_t(total), 0, ring_pages(c, ids[i])};
    total += n_new[i];
    if (total > (int64_t(1) << 30)) return fail(KVQ_ERR_INVALID_ARG, "too many tokens in one append");
  }
  if (total == 0) return KVQ_OK;
  if (!k || !v) return fail(KVQ_ERR_INVALID_ARG, "k or v is NULL");
  if (!aligned16(k) || !aligned16(v)) return fail(KVQ_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  if (kvq_status s = need_device(c)) return s;
  return launched(kvq::launch_append(c->layers[layer], 0, b, int(total), k, v, (cudaStream_t)stream), "append");
}

kvq_status kvq_decode_workspace_size(const kvq_cache* c, int32_t n, int32_t n_q_heads, size_t* bytes) {
  if (kvq_status s = check_cache(c)) return s;
  if (!bytes) return fail(KVQ_ERR_INVALID_ARG, "bytes is NULL");
  if (n < 1 || n > kvq::kMaxBatch) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [1, %d]", kvq::kMaxBatch);
  if (n_q_heads < 1 || n_q_heads % c->L.n_kv_heads) return fail(KVQ_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  const int G = n_q_heads / c->L.n_kv_heads;
  *bytes = kvq::decode_workspace_bytes(n * c->L.n_kv_heads, kvq::decode_max_ctas(c->num_sms), G, c->L.head_dim);
  return KVQ_OK;
}

}  // extern "C"

namespace {

// Argument checks shared by the decode calls (not the layer or the workspace size); *G = the GQA group.
kvq_status decode_check(kvq_cache* c, int32_t n, const int32_t* ids, int32_t n_q_heads, const void* q,
                        const void* k_new, const void* v_new, void* out, float softmax_scale, void* ws, int* G) {
  if (kvq_status s = check_ids(c, n, ids)) return s;
  if (n_q_heads < 1 || n_q_heads % c->L.n_kv_heads) return fail(KVQ_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  *G = n_q_heads / c->L.n_kv_heads;
  if (*G != 1 && *G != 2 && *G != 4 && *G != 8) return fail(KVQ_ERR_UNSUPPORTED, "GQA group %d not built (1, 2, 4, 8)", *G);
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "q or out is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  const bool appending = k_new || v_new;
  if (appending && (!k_new || !v_new)) return fail(KVQ_ERR_INVALID_ARG, "k_new and v_new must both be given");
  if (appending && (!aligned16(k_new) || !aligned16(v_new)))
    return fail(KVQ_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  if (ws && !aligned16(ws)) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return fail(KVQ_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  for (int i = 0; i < n; ++i)
    if (c->len[ids[i]] < 1) return fail(KVQ_ERR_INVALID_ARG, "sequence %d is empty", ids[i]);
  return KVQ_OK;
}

// Layers from `layer` (at most n_layers) that one layer-batched launch takes: consecutive layers
// of the first one's format, whose entries (layers x sequences) fit one batch.
int32_t decode_run_layers(const kvq_cache* c, int32_t layer, int32_t n_layers, int32_t n) {
  const int32_t cap = std::max<int32_t>(1, kvq::kMaxBatch / n);
  int32_t nl = 1;
  while (nl < n_layers && nl < cap && c->k_bits[layer + nl] == c->k_bits[layer] &&
         c->v_bits[layer + nl] == c->v_bits[layer])
    ++nl;
  return nl;
}

// One decode launch over the entries (layer + l, ids[i]) for l < nl, i < n, entry e = l n + i
// (rows of q, out, k_new, v_new in that order); with k_new / v_new, position len - 1 of every
// entry is quantised first (fused into the decode kernel for quantized caches, a separate
// append launch otherwise).  The nl layers share a format (their head blocks lie one layer's
// pool apart), so they are one launch's Layout.  batched: part of a layer-batched call.
// Arguments are checked by the caller.
kvq_status decode_run(kvq_cache* c, int32_t layer, int32_t nl, bool batched, int32_t n, const int32_t* ids, int G,
                      int32_t n_q_heads, const void* q, const void* k_new, const void* v_new, void* out,
                      float softmax_scale, void* ws, kvq_stream_t stream) {
  const bool appending = k_new != nullptr;
  kvq::DecodePlan plan;
  kvq::Layout LV = c->layers[layer];
  bool windowed = false;
  for (int i = 0; i < n; ++i) windowed |= c->window[ids[i]] != 0;
  // rotating windows and layer-batched calls run on the CUDA-core kernels
  if (windowed || batched) LV.decode_tc = 0;
  plan.chunk_tokens = kvq::decode_chunk_tokens(LV, G);
  const int H = c->L.n_kv_heads;
  const int max_ctas = kvq::decode_max_ctas(c->num_sms);
  if (plan.chunk_tokens == 256) {
    // 256-token stages pay off when every CTA gets at least two of them (the consumer overlaps one
    // stage's scores with the previous stage's values); a smaller step keeps 128-token stages
    int64_t n256 = 0;
    for (int i = 0; i < n; ++i) {
      const int64_t len = c->len[ids[i]], lo = first_attended(c, ids[i]);
      n256 += int64_t(nl) * H * ((len - lo / 256 * 256 + 255) / 256);
    }
    if (n256 < 2 * int64_t(max_ctas)) plan.chunk_tokens = 128;
  }
  const int C = plan.chunk_tokens;
  const int ne = nl * n;                             // entries, <= kMaxBatch
  kvq::Batch b;
  b.n = ne;
  int64_t flat = 0;
  int32_t max_nch = 0;
  for (int l = 0; l < nl; ++l)
    for (int i = 0; i < n; ++i) {
      const int64_t len = c->len[ids[i]];
      const int64_t lo = first_attended(c, ids[i]), base = lo / C * C;
      const int32_t nch = int32_t((len - base + C - 1) / C);
      b.s[l * n + i] = {ids[i], int32_t(len), 0, nch, int32_t(lo), ring_pages(c, ids[i]), nch, l};
      flat += int64_t(H) * nch;
      max_nch = std::max(max_nch, nch);
    }
  if (flat >= (int64_t(1) << 31)) return fail(KVQ_ERR_INVALID_ARG, "batch too large");
  // Every CTA takes cpc consecutive chunks of the flat (entry, head, chunk) list.  When the
  // grid still fits in max_ctas, each item is padded to a whole number of CTA ranges, so that no
  // range crosses an item (such a CTA runs two items back to back, each with its own merge), and
  // items of at most kWholeItemChunks chunks go to one CTA whole (nothing to merge across CTAs).
  constexpr int kWholeItemChunks = 4;
  int64_t cpc = (flat + max_ctas - 1) / max_ctas;
  if (!kvq::decode_tc_supported(LV, G)) {
    const int64_t cp = max_nch <= kWholeItemChunks ? std::max<int64_t>(cpc, max_nch) : cpc;
    int64_t pf = 0;
    for (int e = 0; e < ne; ++e) pf += int64_t(H) * ((b.s[e].c + cp - 1) / cp) * cp;
    if (pf / cp <= max_ctas) {
      cpc = cp;
      for (int e = 0; e < ne; ++e) b.s[e].c = int32_t((b.s[e].c + cp - 1) / cp * cp);
    }
  }
  int64_t off = 0;
  for (int e = 0; e < ne; ++e) {
    b.s[e].b = int32_t(off);
    off += int64_t(H) * b.s[e].c;
  }
  plan.n_items = ne * H;
  plan.total_chunks = off;
  plan.max_ctas = max_ctas;
  plan.chunks_per_cta = cpc;
  plan.n_cta = int((off + cpc - 1) / cpc);
  const float sigma = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(c->L.head_dim));
  const float scale_log2 = sigma * 1.4426950408889634f;
  const bool fused = appending && kvq::decode_fuses_append(LV, G);
  if (appending && !fused) {
    kvq::Batch ab;
    ab.n = ne;
    for (int l = 0; l < nl; ++l)
      for (int i = 0; i < n; ++i)
        ab.s[l * n + i] = {ids[i], int32_t(c->len[ids[i]] - 1), 1, l * n + i, 0, ring_pages(c, ids[i]), 0, l};
    if (kvq_status s = launched(kvq::launch_append(LV, 0, ab, ne, k_new, v_new, (cudaStream_t)stream), "append"))
      return s;
  }
  return launched(kvq::launch_decode(LV, 0, b, plan, n_q_heads, q, out, fused ? k_new : nullptr,
                                     fused ? v_new : nullptr, scale_log2, ws, (cudaStream_t)stream),
                  "decode");
}

// kvq_decode_attn, and with k_new / v_new the appending variant.
kvq_status decode_impl(kvq_cache* c, int32_t layer, int32_t n, const int32_t* ids, int32_t n_q_heads, const void* q,
                       const void* k_new, const void* v_new, void* out, float softmax_scale, void* ws,
                       size_t ws_bytes, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_layer(c, layer)) return s;
  int G = 0;
  if (kvq_status s = decode_check(c, n, ids, n_q_heads, q, k_new, v_new, out, softmax_scale, ws, &G)) return s;
  size_t need = 0;
  if (kvq_status s = kvq_decode_workspace_size(c, n, n_q_heads, &need)) return s;
  if (!ws || ws_bytes < need) return fail(KVQ_ERR_WORKSPACE, "decode needs %zu workspace bytes, got %zu", need, ws ? ws_bytes : 0);
  if (kvq_status s = need_device(c)) return s;
  return decode_run(c, layer, 1, false, n, ids, G, n_q_heads, q, k_new, v_new, out, softmax_scale, ws, stream);
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attn(kvq_cache* c, int32_t layer, int32_t n, const int32_t* ids, int32_t n_q_heads,
                           const void* q, void* out, float softmax_scale, void* ws, size_t ws_bytes,
                           kvq_stream_t stream) {
  return decode_impl(c, layer, n, ids, n_q_heads, q, nullptr, nullptr, out, softmax_scale, ws, ws_bytes, stream);
}

kvq_status kvq_decode_append_attn(kvq_cache* c, int32_t layer, int32_t n, const int32_t* ids, int32_t n_q_heads,
                                  const void* q, const void* k_new, const void* v_new, void* out,
                                  float softmax_scale, void* ws, size_t ws_bytes, kvq_stream_t stream) {
  if (!k_new || !v_new) return fail(KVQ_ERR_INVALID_ARG, "k_new or v_new is NULL");
  return decode_impl(c, layer, n, ids, n_q_heads, q, k_new, v_new, out, softmax_scale, ws, ws_bytes, stream);
}

kvq_status kvq_decode_layers_workspace_size(const kvq_cache* c, int32_t n_layers, int32_t n, int32_t n_q_heads,
                                            size_t* bytes) {
  if (kvq_status s = check_cache(c)) return s;
  if (n_layers < 1 || n_layers > c->cfg.n_layers) return fail(KVQ_ERR_INVALID_ARG, "n_layers must be in [1, %d]", c->cfg.n_layers);
  if (n < 1 || n > kvq::kMaxBatch) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [1, %d]", kvq::kMaxBatch);
  // the largest launch: min(n_layers, kMaxBatch / n) layers of the n sequences
  const int32_t nl = std::min<int32_t>(n_layers, std::max<int32_t>(1, kvq::kMaxBatch / n));
  return kvq_decode_workspace_size(c, nl * n, n_q_heads, bytes);
}

kvq_status kvq_decode_attn_layers(kvq_cache* c, int32_t layer0, int32_t n_layers, int32_t n, const int32_t* ids,
                                  int32_t n_q_heads, const void* q, const void* k_new, const void* v_new, void* out,
                                  float softmax_scale, void* ws, size_t ws_bytes, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (layer0 < 0 || n_layers < 1 || int64_t(layer0) + n_layers > c->cfg.n_layers)
    return fail(KVQ_ERR_INVALID_ARG, "layers [%d, %d + %d) outside [0, %d)", layer0, layer0, n_layers, c->cfg.n_layers);
  int G = 0;
  if (kvq_status s = decode_check(c, n, ids, n_q_heads, q, k_new, v_new, out, softmax_scale, ws, &G)) return s;
  size_t need = 0;
  if (kvq_status s = kvq_decode_layers_workspace_size(c, n_layers, n, n_q_heads, &need)) return s;
  if (!ws || ws_bytes < need) return fail(KVQ_ERR_WORKSPACE, "decode needs %zu workspace bytes, got %zu", need, ws ? ws_bytes : 0);
  if (kvq_status s = need_device(c)) return s;
  // rows of one layer in q / out and in k_new / v_new (fp16)
  const int64_t q_layer = int64_t(n) * n_q_heads * c->L.head_dim * 2;
  const int64_t kv_layer = int64_t(n) * c->L.n_kv_heads * c->L.head_dim * 2;
  auto at = [](const void* p, int64_t bytes) -> const void* {
    return p ? static_cast<const void*>(static_cast<const uint8_t*>(p) + bytes) : nullptr;
  };
  for (int32_t l = 0; l < n_layers;) {
    const int32_t nl = decode_run_layers(c, layer0 + l, n_layers - l, n);
    if (kvq_status s = decode_run(c, layer0 + l, nl, true, n, ids, G, n_q_heads, at(q, l * q_layer), at(k_new, l * kv_layer),
                                  at(v_new, l * kv_layer), static_cast<uint8_t*>(out) + l * q_layer, softmax_scale, ws,
                                  stream))
      return s;
    l += nl;
  }
  return KVQ_OK;
}

kvq_status kvq_prefill_workspace_size(const kvq_cache* c, int32_t n, const int32_t* ids, const int32_t* q_lens,
                                      int32_t n_q_heads, size_t* bytes) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_ids(c, n, ids)) return s;
  if (!q_lens || !bytes) return fail(KVQ_ERR_INVALID_ARG, "q_lens or bytes is NULL");
  if (n_q_heads < 1 || n_q_heads % c->L.n_kv_heads) return fail(KVQ_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  kvq::Batch b;
  b.n = n;
  int64_t total = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t len = c->len[ids[i]];
    if (q_lens[i] < 1 || q_lens[i] > len) return fail(KVQ_ERR_INVALID_ARG, "q_lens[%d] outside [1, len]", i);
    b.s[i] = {ids[i], int32_t(len), q_lens[i], int32_t(total)};
    total += q_lens[i];
  }
  *bytes = kvq::prefill_workspace_bytes(c->L, b);
  return KVQ_OK;
}

kvq_status kvq_prefill_attn(kvq_cache* c, int32_t layer, int32_t n, const int32_t* ids, const int32_t* q_lens,
                            int32_t n_q_heads, const void* q, void* out, float softmax_scale, void* ws,
                            size_t ws_bytes, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_layer(c, layer)) return s;
  if (kvq_status s = check_ids(c, n, ids)) return s;
  if (!q_lens) return fail(KVQ_ERR_INVALID_ARG, "q_lens is NULL");
  if (n_q_heads < 1 || n_q_heads % c->L.n_kv_heads) return fail(KVQ_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  const int G = n_q_heads / c->L.n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(KVQ_ERR_UNSUPPORTED, "GQA group %d not built (1, 2, 4, 8)", G);
  if (c->L.head_dim != 128 && c->L.head_dim != 64) return fail(KVQ_ERR_UNSUPPORTED, "head_dim not built for prefill");
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "q or out is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  if (ws && !aligned16(ws)) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return fail(KVQ_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  kvq::Batch b;
  b.n = n;
  int64_t total = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t len = c->len[ids[i]];
    if (q_lens[i] < 1 || q_lens[i] > len) return fail(KVQ_ERR_INVALID_ARG, "q_lens[%d] outside [1, len]", i);
    if (c->window[ids[i]] && len > c->window[ids[i]])
      return fail(KVQ_ERR_UNSUPPORTED, "prefill of sequence %d beyond its rotating window", ids[i]);
    b.s[i] = {ids[i], int32_t(len), q_lens[i], int32_t(total)};
    total += q_lens[i];
    if (total > (int64_t(1) << 30)) return fail(KVQ_ERR_INVALID_ARG, "too many query rows");
  }
  const size_t need = kvq::prefill_workspace_bytes(c->L, b);
  if (need && (!ws || ws_bytes < need))
    return fail(KVQ_ERR_WORKSPACE, "prefill needs %zu workspace bytes, got %zu", need, ws ? ws_bytes : 0);
  if (kvq_status s = need_device(c)) return s;
  const float sigma = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(c->L.head_dim));
  return launched(kvq::launch_prefill(c->layers[layer], 0, b, int(total), n_q_heads, q, out, sigma, ws, ws_bytes,
                                      c->pstreams, (cudaStream_t)stream),
                  "prefill");
}

kvq_status kvq_cache_dedup(kvq_cache* c, kvq_stream_t stream, int64_t* pages_freed) {
  if (kvq_status s = check_cache(c)) return s;
  if (pages_freed) *pages_freed = 0;
  if (kvq_status s = need_device(c)) return s;
  const int P = c->L.page_tokens, L = c->cfg.n_layers;
  const int32_t mpps = c->L.max_pages_per_seq;
  cudaStream_t st = (cudaStream_t)stream;
  // candidates: pages every mapping of which is a full page of a sequence without a window
  std::vector<int8_t> state(c->L.n_pages, 0);                 // 0 unseen, 1 candidate, -1 excluded
  std::vector<std::vector<int32_t>> slots_of;                  // mapping slots per candidate, filled below
  for (int32_t id = 0; id < c->cfg.max_seqs; ++id)
    for (int32_t p = 0; p < c->mapped[id]; ++p) {
      const int32_t phys = c->table[size_t(id) * mpps + p];
      const bool full = !c->window[id] && int64_t(p + 1) * P <= c->len[id];
      if (!full) state[phys] = -1;
      else if (state[phys] == 0) state[phys] = 1;
    }
  std::vector<int32_t> cand;
  std::vector<int32_t> index(c->L.n_pages, -1);
  for (int32_t pg = 0; pg < c->L.n_pages; ++pg)
    if (state[pg] == 1) {
      index[pg] = int32_t(cand.size());
      cand.push_back(pg);
    }
  if (cand.size() < 2) return KVQ_OK;
  slots_of.resize(cand.size());
  for (int32_t id = 0; id < c->cfg.max_seqs; ++id)
    for (int32_t p = 0; p < c->mapped[id]; ++p) {
      const size_t slot = size_t(id) * mpps + p;
      if (index[c->table[slot]] >= 0) slots_of[index[c->table[slot]]].push_back(int32_t(slot));
    }
  auto regions = [&](kvq::PageRegion* out, int l0, int nl) {
    for (int l = 0; l < nl; ++l) {
      const kvq::Layout& V = c->layers[l0 + l];
      out[l] = {V.pool, int64_t(V.n_kv_heads) * V.head_block};
    }
  };
  // 128-bit content hashes, kDedupBatch pages at a time
  std::vector<std::array<uint32_t, 4>> hash(cand.size());
  uint32_t* d_hash = c->d_dedup;
  uint32_t* d_diff = c->d_dedup + 4 * kvq::kDedupBatch;
  kvq::PageList pl;
  for (size_t b0 = 0; b0 < cand.size(); b0 += kvq::kDedupBatch) {
    pl.n = int32_t(std::min<size_t>(kvq::kDedupBatch, cand.size() - b0));
    for (int i = 0; i < pl.n; ++i) pl.page[i] = cand[b0 + i];
    for (int l0 = 0; l0 < L; l0 += kvq::kDedupLayers) {
      const int nl = std::min(kvq::kDedupLayers, L - l0);
      regions(pl.layer, l0, nl);
      KVQ_CUDA(kvq::launch_page_hash(pl, nl, d_hash, l0 == 0, st), "page hash");
    }
    KVQ_CUDA(cudaMemcpyAsync(hash[b0].data(), d_hash, size_t(pl.n) * 16, cudaMemcpyDeviceToHost, st), "read hashes");
    KVQ_CUDA(cudaStreamSynchronize(st), "page hash");
  }
  // equal hashes propose duplicates of the group's first page; a byte comparison decides
  std::vector<int32_t> order(cand.size());
  for (size_t i = 0; i < cand.size(); ++i) order[i] = int32_t(i);
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) { return hash[x] < hash[y]; });
  std::vector<std::pair<int32_t, int32_t>> pairs;                 // (representative, duplicate) candidate indices
  for (size_t i = 0; i < order.size();) {
    size_t j = i + 1;
    while (j < order.size() && hash[order[j]] == hash[order[i]]) ++j;
    for (size_t k = i + 1; k < j; ++k) pairs.push_back({order[i], order[k]});
    i = j;
  }
  std::vector<uint8_t> same(pairs.size(), 0);
  kvq::PagePairs pp;
  std::vector<uint32_t> diff(kvq::kDedupBatch);
  for (size_t b0 = 0; b0 < pairs.size(); b0 += kvq::kDedupBatch) {
    pp.n = int32_t(std::min<size_t>(kvq::kDedupBatch, pairs.size() - b0));
    for (int i = 0; i < pp.n; ++i) {
      pp.a[i] = cand[pairs[b0 + i].first];
      pp.b[i] = cand[pairs[b0 + i].second];
    }
    for (int l0 = 0; l0 < L; l0 += kvq::kDedupLayers) {
      const int nl = std::min(kvq::kDedupLayers, L - l0);
      regions(pp.layer, l0, nl);
      KVQ_CUDA(kvq::launch_page_compare(pp, nl, d_diff, l0 == 0, st), "page compare");
    }
    KVQ_CUDA(cudaMemcpyAsync(diff.data(), d_diff, size_t(pp.n) * 4, cudaMemcpyDeviceToHost, st), "read compare");
    KVQ_CUDA(cudaStreamSynchronize(st), "page compare");
    for (int i = 0; i < pp.n; ++i) same[b0 + i] = diff[i] == 0;
  }
  // merge: every slot mapping a duplicate maps its representative instead
  Journal j;
  kvq::PtUpdate upd;
  upd.n = 0;
  size_t flushed = 0;
  kvq_status stt = KVQ_OK;
  int64_t freed = 0;
  for (size_t k = 0; k < pairs.size() && stt == KVQ_OK; ++k) {
    if (!same[k]) continue;
    const int32_t rep = cand[pairs[k].first], dup = cand[pairs[k].second];
    for (int32_t slot : slots_of[pairs[k].second]) {
      set_slot(c, size_t(slot), rep, &j);
      c->refs[rep]++;
      j.add(Journal::kRef, rep);
      drop_page(c, dup, &j);
      upd.idx[upd.n] = slot;
      upd.val[upd.n] = rep;
      if (++upd.n == kvq::kMaxPtUpdates) {
        stt = launched(kvq::launch_pt_update(c->d_page_table, upd, st), "page-table update");
        if (stt == KVQ_OK) flushed = j.ops.size();
        upd.n = 0;
        if (stt != KVQ_OK) break;
      }
    }
    ++freed;
  }
  if (stt == KVQ_OK && upd.n) {
    stt = launched(kvq::launch_pt_update(c->d_page_table, upd, st), "page-table update");
    if (stt == KVQ_OK) flushed = j.ops.size();
  }
  if (stt != KVQ_OK) {
    rollback(c, j, flushed, stream);
    return stt;
  }
  if (pages_freed) *pages_freed = freed;
  return KVQ_OK;
}

kvq_status kvq_export(const kvq_cache* c, int32_t layer, int32_t id, int64_t tok0, int64_t n_tok, void* kc,
                      void* ks, void* vc, void* vs, kvq_stream_t stream) {
  if (kvq_status s = check_cache(c)) return s;
  if (kvq_status s = check_layer(c, layer)) return s;
  if (kvq_status s = check_seq(c, id)) return s;
  if (tok0 < 0 || n_tok < 0 || tok0 + n_tok > c->len[id]) return fail(KVQ_ERR_INVALID_ARG, "token range outside the sequence");
  if (c->window[id] && tok0 < c->len[id] - c->window[id])
    return fail(KVQ_ERR_INVALID_ARG, "token range starts before the sequence's rotating window");
  if (n_tok == 0) return KVQ_OK;
  if (kvq_status s = need_device(c)) return s;
  return launched(kvq::launch_export(c->layers[layer], 0, id, ring_pages(c, id), tok0, n_tok, kc, ks, vc, vs,
                                     (cudaStream_t)stream),
                  "export");
}

kvq_status kvq_cache_check(kvq_cache* c, kvq_stream_t stream, uint32_t* detail) {
  if (kvq_status s = check_cache(c)) return s;
  if (detail) *detail = 0;
  if (c->host_only) return KVQ_OK;
  if (kvq_status s = same_device(c)) return s;
  KVQ_CUDA(cudaStreamSynchronize((cudaStream_t)stream), "cudaStreamSynchronize");
  KVQ_CUDA(cudaGetLastError(), "earlier launch");
  uint32_t code = 0;
  KVQ_CUDA(cudaMemcpy(&code, c->d_err, sizeof code, cudaMemcpyDeviceToHost), "read device error word");
  if (code) {
    if (detail) *detail = code;
    KVQ_CUDA(cudaMemset(c->d_err, 0, sizeof code), "clear device error word");
    // a kernel that gave up may have left split-item counters raised
    KVQ_CUDA(cudaMemset(c->d_counters, 0, size_t(kvq::kMaxBatch) * c->L.n_kv_heads * sizeof(int32_t)),
             "clear decode counters");
    return fail(KVQ_ERR_DEVICE_CHECK, "device check failed, code 0x%x", code);
  }
  return KVQ_OK;
}

}  // extern "C"
