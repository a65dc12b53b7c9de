"""Host-side tests of the C-ABI library (no GPU needed): exported symbols, the
library's footprint closed form against the KVSplit page's table, the page
allocator and argument validation on a host-only cache."""
import ctypes
import os
import re

import pytest

from asymmetric_quantized_kv_kvq_b200 import build as kbuild
from oracle import footprint_bytes as oracle_footprint, footprint_bytes_layers

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    kbuild.build()
    from asymmetric_quantized_kv_kvq_b200 import kvq as m
    m.load_library()
    return m


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "kvq.h")) as f:
        text = f.read()
    return set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text))


def test_header_symbols_are_exported(kvq):
    declared = _declared_symbols()
    assert len(declared) >= 17
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    # the binding marshals exactly the declared calls
    assert declared == set(kvq.SIGNATURES)


def test_status_strings(kvq):
    lib = kvq.load_library()
    for code in range(8):
        assert lib.kvq_status_string(code)
    assert lib.kvq_status_string(0) == b"ok"


BITS = {"FP16": (16, 16), "K8V8": (8, 8), "K8V4": (8, 4), "K4V8": (4, 8), "K4V4": (4, 4)}


@pytest.mark.parametrize("cfg", list(BITS))
@pytest.mark.parametrize("tokens", [1, 128, 255, 256, 257, 4096, 8192, 100000])
def test_library_footprint_matches_oracle(kvq, cfg, tokens):
    kb, vb = BITS[cfg]
    alloc, used = kvq.footprint_bytes(22, 4, 64, kb, vb, tokens)
    assert alloc == oracle_footprint(22, 4, 64, kb, vb, tokens)
    assert used == 22 * tokens * (alloc // (22 * (-(-tokens // 256)) * 256))


def test_library_footprint_reproduces_the_printed_table(kvq):
    mib = 1 << 20
    want = {("FP16", 8192): 176.00, ("K8V8", 8192): 93.50, ("K8V4", 8192): 71.50, ("K4V4", 8192): 49.50,
            ("FP16", 4096): 88.00, ("K8V4", 4096): 35.75, ("K4V4", 4096): 24.75,
            ("FP16", 128): 5.50, ("K8V4", 128): 2.23, ("K4V4", 128): 1.55}
    for (cfg, tokens), v in want.items():
        kb, vb = BITS[cfg]
        assert round(kvq.footprint_bytes(22, 4, 64, kb, vb, tokens)[0] / mib, 2) == v


def _host_cache(kvq, **kw):
    args = dict(n_layers=2, n_kv_heads=2, head_dim=64, k_bits=8, v_bits=4, max_seqs=4, max_tokens=1024,
                page_tokens=256, host_only=True)
    args.update(kw)
    return kvq.Cache(**args)


def test_host_only_allocator(kvq):
    c = _host_cache(kvq)
    pool, mapped, used = c.footprint()
    per_tok = 2 * 2 * (64 + 4 + 32 + 4)          # layers * heads * (K8 + V4 bytes)
    assert pool == 4 * 256 * per_tok and mapped == 0 and used == 0
    c.extend([0, 1], [1, 300])
    assert c.length(0) == 1 and c.length(1) == 300
    assert c.page(0, 0) == 0 and c.page(1, 0) == 1 and c.page(1, 1) == 2 and c.page(1, 2) == -1
    assert c.footprint()[1] == 3 * 256 * per_tok
    assert c.footprint()[2] == 301 * per_tok
    c.extend([0], [255])                           # fills page 0 exactly
    assert c.page(0, 1) == -1 and c.length(0) == 256
    c.extend([0], [1])
    assert c.page(0, 1) == 3
    # pool exhausted: all-or-nothing
    with pytest.raises(kvq.KvqError) as e:
        c.extend([2, 3], [1, 1])
    assert e.value.name == "KVQ_ERR_CAPACITY"
    assert c.length(2) == 0 and c.length(3) == 0
    c.release(1)
    assert c.length(1) == 0 and c.page(1, 0) == -1
    c.extend([2], [512])                            # reuses the two released pages
    assert sorted([c.page(2, 0), c.page(2, 1)]) == [1, 2]
    c.close()


def test_truncate_returns_whole_pages(kvq):
    c = _host_cache(kvq)
    c.extend([0], [600])                         # pages 0, 1, 2
    assert [c.page(0, i) for i in range(3)] == [0, 1, 2]
    c.truncate(0, 300)                           # keeps 2 pages
    assert c.length(0) == 300 and c.page(0, 2) == -1
    c.truncate(0, 256)                           # exactly one page
    assert c.page(0, 1) == -1 and c.page(0, 0) == 0
    with pytest.raises(kvq.KvqError):
        c.truncate(0, 257)                       # cannot grow
    c.extend([0], [1])                           # the next page is the last one freed
    assert c.page(0, 1) == 1
    c.truncate(0, 0)
    assert c.footprint()[1] == 0 and c.length(0) == 0
    c.close()


def test_fork_shares_pages_and_copies_a_shared_tail_before_writing(kvq):
    c = _host_cache(kvq, max_tokens=2048)                 # 8 pages
    per_page = 2 * 2 * (64 + 4 + 32 + 4) * 256
    c.extend([0], [300])                                  # pages 0, 1 (page 1 partly filled)
    c.fork(0, 1)                                          # seq 1 = all 300 positions of seq 0
    assert c.length(1) == 300 and [c.page(1, i) for i in range(2)] == [0, 1]
    assert c.footprint()[1] == 2 * per_page               # shared pages count once
    c.extend([0, 1], [1, 1])                              # both write into page 1: seq 0 copies it first
    assert c.page(0, 0) == 0 and c.page(1, 0) == 0        # the full page stays shared
    assert c.page(0, 1) == 2 and c.page(1, 1) == 1        # seq 1 is now the only user of page 1
    assert c.footprint()[1] == 3 * per_page
    c.fork(0, 2, 256)                                     # a page-aligned prefix: nothing to copy later
    c.extend([2], [10])
    assert c.page(2, 0) == 0 and c.page(2, 1) == 3
    c.fork(1, 3, 100)                                     # a prefix ending inside shared page 0
    c.extend([3], [1])                                    # page 0 is copied for seq 3 before the write
    assert c.page(3, 0) == 4 and c.page(0, 0) == 0 and c.length(3) == 101
    c.release(0)
    c.release(2)
    assert c.page(1, 0) == 0                              # still held by seq 1
    c.release(1)
    c.release(3)
    assert c.footprint()[1] == 0
    c.extend([0], [2048])                                 # every page is free again
    with pytest.raises(kvq.KvqError) as e:
        c.fork(0, 0)
    assert e.value.name == "KVQ_ERR_INVALID_ARG"
    c.extend([1], [0])
    with pytest.raises(kvq.KvqError):
        c.fork(0, 1, 2049)                                # longer than the source
    c.close()


def test_fork_respects_the_capacity_check(kvq):
    c = _host_cache(kvq, max_tokens=768)                  # 3 pages
    c.extend([0], [300])                                  # pages 0, 1; one free
    c.fork(0, 1)
    with pytest.raises(kvq.KvqError) as e:
        c.extend([0, 1], [1, 1])
    # a copy is counted for each sequence whose last page is shared, although the second one would find
    # the page private by then: the check is conservative, and nothing changes
    assert e.value.name == "KVQ_ERR_CAPACITY"
    assert c.length(0) == 300 and c.length(1) == 300 and c.page(0, 1) == c.page(1, 1) == 1
    c.extend([1], [1])                                    # one copy fits
    assert c.page(1, 1) == 2 and c.page(0, 1) == 1 and c.length(1) == 301
    with pytest.raises(kvq.KvqError) as e:                # no page left for a copy
        c.fork(1, 2)
        c.fork(1, 3)
        c.extend([2], [1])
    assert e.value.name == "KVQ_ERR_CAPACITY"
    c.close()


def test_max_seq_tokens_bound(kvq):
    c = _host_cache(kvq, max_seq_tokens=300)
    c.extend([0], [300])
    with pytest.raises(kvq.KvqError) as e:
        c.extend([0], [1])
    assert e.value.name == "KVQ_ERR_CAPACITY"
    c.close()


@pytest.mark.parametrize("kw,name", [
    (dict(k_bits=3), "KVQ_ERR_INVALID_ARG"),
    (dict(head_dim=48), "KVQ_ERR_INVALID_ARG"),
    (dict(head_dim=96), "KVQ_ERR_UNSUPPORTED"),
    (dict(k_bits=16, v_bits=4), "KVQ_ERR_UNSUPPORTED"),
    (dict(page_tokens=100), "KVQ_ERR_INVALID_ARG"),
    (dict(max_seqs=0), "KVQ_ERR_INVALID_ARG"),
    (dict(max_tokens=0), "KVQ_ERR_INVALID_ARG"),
    (dict(n_layers=0), "KVQ_ERR_INVALID_ARG"),
])
def test_bad_configs(kvq, kw, name):
    with pytest.raises(kvq.KvqError) as e:
        _host_cache(kvq, **kw)
    assert e.value.name == name


def test_bad_calls_leave_the_cache_unchanged(kvq):
    c = _host_cache(kvq)
    c.extend([0], [10])
    lib = kvq.load_library()
    ids = (ctypes.c_int32 * 2)(0, 0)
    n = (ctypes.c_int32 * 2)(1, 1)
    assert lib.kvq_seq_extend(c._h, 2, ids, n, None) == 1          # repeated id
    ids1 = (ctypes.c_int32 * 1)(9)
    assert lib.kvq_seq_extend(c._h, 1, ids1, n, None) == 1         # unknown id
    assert lib.kvq_seq_extend(c._h, 0, ids1, n, None) == 1         # empty batch
    neg = (ctypes.c_int32 * 1)(-1)
    ids0 = (ctypes.c_int32 * 1)(0)
    assert lib.kvq_seq_extend(c._h, 1, ids0, neg, None) == 1       # negative count
    assert c.length(0) == 10
    # append: layer out of range, more new tokens than the length, NULL data
    n11 = (ctypes.c_int32 * 1)(11)
    one = (ctypes.c_int32 * 1)(1)
    assert lib.kvq_append(c._h, 2, 1, ids0, one, 1, 1, None) == 1
    assert lib.kvq_append(c._h, 0, 1, ids0, n11, 1, 1, None) == 1
    assert lib.kvq_append(c._h, 0, 1, ids0, one, None, None, None) == 1
    # decode: bad head grouping, GQA group not built, missing workspace, host-only
    assert lib.kvq_decode_attn(c._h, 0, 1, ids0, 3, 16, 16, 0.0, 16, 1 << 20, None) == 1
    assert lib.kvq_decode_attn(c._h, 0, 1, ids0, 6, 16, 16, 0.0, 16, 1 << 20, None) == 2
    assert lib.kvq_decode_attn(c._h, 0, 1, ids0, 4, 16, 16, 0.0, None, 0, None) == 7
    assert lib.kvq_decode_attn(c._h, 0, 1, ids0, 4, 16, 16, -1.0, 16, 1 << 20, None) == 1
    assert lib.kvq_decode_attn(c._h, 0, 1, ids0, 4, 16, 16, 0.0, 16, 1 << 20, None) == 2
    assert lib.kvq_decode_attn(c._h, 0, 1, ids0, 4, 8, 16, 0.0, 16, 1 << 20, None) == 1
    # export beyond the length
    assert lib.kvq_export(c._h, 0, 0, 5, 6, 1, 1, 1, 1, None) == 1
    # prefill: chunk longer than the sequence
    assert lib.kvq_prefill_attn(c._h, 0, 1, ids0, n11, 4, 1, 1, 0.0, None, 0, None) == 1
    assert c.length(0) == 10
    assert b"out of range" in lib.kvq_last_error() or lib.kvq_last_error()
    c.close()


def test_decode_workspace_is_length_independent(kvq):
    c = _host_cache(kvq)
    a = c.decode_workspace_size(1, 4)
    b = c.decode_workspace_size(2, 4)
    assert 0 < a < b
    with pytest.raises(kvq.KvqError):
        c.decode_workspace_size(0, 4)
    with pytest.raises(kvq.KvqError):
        c.decode_workspace_size(300, 4)
    c.close()


def test_destroy_null_is_noop(kvq):
    assert kvq.load_library().kvq_cache_destroy(None) == 0


def test_cache_flags(kvq):
    """The header's flag values, and unknown bits refused before anything is allocated."""
    with open(os.path.join(ROOT, "include", "kvq.h")) as f:
        text = f.read()
    assert re.search(r"#define KVQ_CACHE_HOST_ONLY 1\b", text)
    assert re.search(r"#define KVQ_CACHE_DECODE_TENSOR_CORES 2\b", text)
    assert kvq.KVQ_CACHE_HOST_ONLY == 1 and kvq.KVQ_CACHE_DECODE_TENSOR_CORES == 2
    lib = kvq.load_library()
    cfg = kvq.make_config(1, 8, 128, 8, 4, 2, 4096, host_only=True, decode_tc=True)
    assert cfg.flags == 3
    h = ctypes.c_void_p()
    assert lib.kvq_cache_create(ctypes.byref(cfg), ctypes.byref(h)) == 0
    assert lib.kvq_cache_destroy(h) == 0
    cfg.flags = 1 | 4
    h = ctypes.c_void_p()
    assert lib.kvq_cache_create(ctypes.byref(cfg), ctypes.byref(h)) == 1      # KVQ_ERR_INVALID_ARG
    assert b"unknown flags" in lib.kvq_last_error()


def test_injected_allocation_failure_is_reported_and_cleaned_up(kvq, monkeypatch):
    """Host-side fault injection: a failed bookkeeping allocation returns KVQ_ERR_OUT_OF_MEMORY with no
    cache created, and the next creation succeeds."""
    monkeypatch.setenv("KVQ_INJECT_ALLOC_FAILURE", "1")
    with pytest.raises(kvq.KvqError) as e:
        _host_cache(kvq)
    assert e.value.name == "KVQ_ERR_OUT_OF_MEMORY"
    monkeypatch.delenv("KVQ_INJECT_ALLOC_FAILURE")
    c = _host_cache(kvq)
    c.extend([0], [10])
    assert c.length(0) == 10
    c.close()


def _allocator_state(c, ids, pages):
    return ([c.length(i) for i in ids], [[c.page(i, p) for p in range(pages)] for i in ids], c.footprint())


@pytest.mark.parametrize("nth", [1, 2])
def test_extend_is_all_or_nothing_when_a_page_table_enqueue_fails(kvq, monkeypatch, nth):
    """Host-side fault injection: the nth page-table enqueue of kvq_seq_extend fails (the first one after
    1024 updates, or the final one).  The call returns KVQ_ERR_CUDA and no sequence, page or reference
    changes; the same extend then succeeds and hands out the pages a fresh cache would."""
    c = kvq.Cache(n_layers=1, n_kv_heads=2, head_dim=64, k_bits=8, v_bits=4, max_seqs=3,
                  max_tokens=64 * 3000, page_tokens=64, host_only=True)
    c.extend([0], [100])
    c.fork(0, 2, 70)                                    # a shared, partly filled tail page (copy-on-write)
    before = _allocator_state(c, [0, 1, 2], 1200)
    monkeypatch.setenv("KVQ_INJECT_PT_FAILURE", str(nth))
    with pytest.raises(kvq.KvqError) as e:
        c.extend([2, 1], [5, 64 * 1100])                # 1 copy-on-write page + 1100 new pages
    assert e.value.name == "KVQ_ERR_CUDA" and "injected" in str(e.value)
    assert _allocator_state(c, [0, 1, 2], 1200) == before
    monkeypatch.delenv("KVQ_INJECT_PT_FAILURE")
    c.extend([2, 1], [5, 64 * 1100])
    fresh = kvq.Cache(n_layers=1, n_kv_heads=2, head_dim=64, k_bits=8, v_bits=4, max_seqs=3,
                      max_tokens=64 * 3000, page_tokens=64, host_only=True)
    fresh.extend([0], [100])
    fresh.fork(0, 2, 70)
    fresh.extend([2, 1], [5, 64 * 1100])
    assert _allocator_state(c, [0, 1, 2], 1200) == _allocator_state(fresh, [0, 1, 2], 1200)
    c.close()
    fresh.close()


def test_fork_is_all_or_nothing_when_a_page_table_enqueue_fails(kvq, monkeypatch):
    """A fork of 1100 pages whose second page-table enqueue fails leaves both sequences and every
    reference count as they were: releasing the source afterwards frees all its pages."""
    c = kvq.Cache(n_layers=1, n_kv_heads=2, head_dim=64, k_bits=8, v_bits=4, max_seqs=2,
                  max_tokens=64 * 1200, page_tokens=64, host_only=True)
    c.extend([0], [64 * 1100])
    before = _allocator_state(c, [0, 1], 1100)
    monkeypatch.setenv("KVQ_INJECT_PT_FAILURE", "2")
    with pytest.raises(kvq.KvqError):
        c.fork(0, 1)
    monkeypatch.delenv("KVQ_INJECT_PT_FAILURE")
    assert _allocator_state(c, [0, 1], 1100) == before
    c.release(0)
    assert c.footprint()[1] == 0                        # no page kept alive by a leaked reference
    c.close()


@pytest.mark.parametrize("tokens", [1, 255, 256, 8192, 100000])
def test_per_layer_precision_footprint_matches_oracle(kvq, tokens):
    bits = [(8, 4), (4, 8), (16, 16), (8, 8), (4, 4), (8, 4)]
    alloc, used = kvq.footprint_bytes(6, 4, 64, 8, 4, tokens, layer_bits=bits)
    assert alloc == footprint_bytes_layers(4, 64, bits, tokens)
    c = kvq.Cache(6, 4, 64, 8, 4, max_seqs=2, max_tokens=tokens + 512, host_only=True, layer_bits=bits)
    c.extend([0], [tokens])
    pool, mapped, used_c = c.footprint()
    assert mapped == alloc and used_c == used
    c.close()


def test_per_layer_precision_validation(kvq):
    lib = kvq.load_library()
    cfg = kvq.make_config(3, 2, 64, 8, 4, 2, 1024, host_only=True, layer_bits=[(8, 4), (16, 8), (4, 4)])
    h = ctypes.c_void_p()
    assert lib.kvq_cache_create(ctypes.byref(cfg), ctypes.byref(h)) == 2      # K16V8 not built
    assert b"layer 1" in lib.kvq_last_error()
    cfg = kvq.make_config(3, 2, 64, 8, 4, 2, 1024, host_only=True, layer_bits=[(8, 4), (8, 3), (4, 4)])
    assert lib.kvq_cache_create(ctypes.byref(cfg), ctypes.byref(h)) == 1
    cfg = kvq.make_config(3, 2, 64, 8, 4, 2, 1024, host_only=True)
    cfg.layer_k_bits = (ctypes.c_int32 * 3)(8, 8, 8)                           # one array without the other
    assert lib.kvq_cache_create(ctypes.byref(cfg), ctypes.byref(h)) == 1
    with pytest.raises(kvq.KvqError):
        kvq.make_config(3, 2, 64, 8, 4, 2, 1024, layer_bits=[(8, 4)])


def test_rotating_window_keeps_a_ring_of_pages(kvq):
    """A 256-token window with 64-token pages keeps a ring of 5 page-table slots: after 1000 one-token
    extends the sequence maps exactly 5 distinct pages in slots 0..4 and nothing beyond; a linear
    sequence next to it maps all its pages; release returns the ring."""
    c = kvq.Cache(n_layers=2, n_kv_heads=2, head_dim=64, k_bits=8, v_bits=4, max_seqs=3, max_tokens=64 * 40,
                  page_tokens=64, max_seq_tokens=64 * 8, host_only=True)
    c.set_window(0, 256)
    for _ in range(1000):
        c.extend([0], [1])
    assert c.length(0) == 1000
    ring = [c.page(0, s) for s in range(8)]
    assert all(p >= 0 for p in ring[:5]) and ring[5:] == [-1, -1, -1] and len(set(ring[:5])) == 5
    pool, mapped, used = c.footprint()
    assert mapped == 5 * 64 * 2 * 2 * (68 + 36)                   # 5 pages x 64 tokens x 2 layers x 2 heads
    c.extend([1], [300])
    assert c.footprint()[1] == (5 + 5) * 64 * 2 * 2 * (68 + 36)
    # a multi-token extend across the ring's wrap point reuses slots in order
    c.extend([0], [200])
    assert [c.page(0, s) for s in range(5)] == ring[:5]
    c.release(0)
    assert c.footprint()[1] == 5 * 64 * 2 * 2 * (68 + 36)
    c.close()


def test_rotating_window_refusals(kvq):
    c = kvq.Cache(n_layers=1, n_kv_heads=2, head_dim=64, k_bits=8, v_bits=4, max_seqs=3, max_tokens=64 * 40,
                  page_tokens=64, max_seq_tokens=64 * 8, host_only=True)
    for bad, name in ((100, "KVQ_ERR_INVALID_ARG"), (-64, "KVQ_ERR_INVALID_ARG"), (512, "KVQ_ERR_CAPACITY")):
        with pytest.raises(kvq.KvqError) as e:
            c.set_window(0, bad)
        assert e.value.name == name
    c.set_window(0, 128)
    c.extend([0], [1000])                                         # windowed: not bounded by max_seq_tokens
    with pytest.raises(kvq.KvqError) as e:
        c.set_window(0, 256)                                      # only on an empty sequence
    assert e.value.name == "KVQ_ERR_INVALID_ARG"
    with pytest.raises(kvq.KvqError) as e:
        c.fork(0, 1, 10)
    assert e.value.name == "KVQ_ERR_UNSUPPORTED"
    with pytest.raises(kvq.KvqError) as e:
        c.truncate(0, 900)
    assert e.value.name == "KVQ_ERR_UNSUPPORTED"
    lib = kvq.load_library()
    ids = (ctypes.c_int32 * 1)(0)
    nn = (ctypes.c_int32 * 1)(129)
    assert lib.kvq_append(c._h, 0, 1, ids, nn, 16, 16, None) == 1    # more than the window in one append
    with pytest.raises(kvq.KvqError):
        c.extend([1], [64 * 8 + 1])                               # a linear sequence keeps its bound
    c.close()


def test_dedup_needs_a_device(kvq):
    c = _host_cache(kvq)
    c.extend([0], [600])
    lib = kvq.load_library()
    n = ctypes.c_int64(-1)
    assert lib.kvq_cache_dedup(c._h, None, ctypes.byref(n)) == 2     # KVQ_ERR_UNSUPPORTED on a host-only cache
    assert n.value == 0
    c.close()


def test_layer_batched_decode_validation_and_workspace(kvq):
    """kvq_decode_attn_layers checks its layer range before anything else and sizes its workspace
    for the largest launch: min(n_layers, KVQ_MAX_BATCH // n_seqs) layers of the batch."""
    c = _host_cache(kvq, n_layers=6, max_seqs=256, max_tokens=256 * 256)
    c.extend([0], [10])
    lib = kvq.load_library()
    ids0 = (ctypes.c_int32 * 1)(0)
    # one sequence: every layer fits one launch, so the workspace is that of 6 entries
    assert c.decode_layers_workspace_size(6, 1, 4) == c.decode_workspace_size(6, 4)
    assert c.decode_layers_workspace_size(1, 1, 4) == c.decode_workspace_size(1, 4)
    # 64 sequences: 4 layers per launch (256 entries); 256 sequences: one layer per launch
    assert c.decode_layers_workspace_size(5, 64, 4) == c.decode_workspace_size(256, 4)
    assert c.decode_layers_workspace_size(3, 64, 4) == c.decode_workspace_size(192, 4)
    assert c.decode_layers_workspace_size(6, 256, 4) == c.decode_workspace_size(256, 4)
    for bad in ((0, 1), (7, 1), (2, 0), (2, 257)):
        with pytest.raises(kvq.KvqError):
            c.decode_layers_workspace_size(bad[0], bad[1], 4)
    ws = 1 << 20
    call = lib.kvq_decode_attn_layers
    # layer range: negative start, empty, past the last layer
    assert call(c._h, -1, 1, 1, ids0, 4, 16, None, None, 16, 0.0, 16, ws, None) == 1
    assert call(c._h, 0, 0, 1, ids0, 4, 16, None, None, 16, 0.0, 16, ws, None) == 1
    assert call(c._h, 4, 3, 1, ids0, 4, 16, None, None, 16, 0.0, 16, ws, None) == 1
    # heads, GQA group, one of k_new / v_new, alignment, workspace, host-only
    assert call(c._h, 0, 6, 1, ids0, 3, 16, None, None, 16, 0.0, 16, ws, None) == 1
    assert call(c._h, 0, 6, 1, ids0, 6, 16, None, None, 16, 0.0, 16, ws, None) == 2
    assert call(c._h, 0, 6, 1, ids0, 4, 16, 16, None, 16, 0.0, 16, ws, None) == 1
    assert call(c._h, 0, 6, 1, ids0, 4, 8, None, None, 16, 0.0, 16, ws, None) == 1
    assert call(c._h, 0, 6, 1, ids0, 4, 16, None, None, 16, 0.0, None, 0, None) == 7
    assert call(c._h, 0, 6, 1, ids0, 4, 16, None, None, 16, 0.0, 16, 16, None) == 7
    assert call(c._h, 0, 6, 1, ids0, 4, 16, 16, 16, 16, 0.0, 16, ws, None) == 2
    # an empty sequence
    ids1 = (ctypes.c_int32 * 1)(1)
    assert call(c._h, 0, 6, 1, ids1, 4, 16, None, None, 16, 0.0, 16, ws, None) == 1
    assert c.length(0) == 10
    c.close()
