"""GPU parity of content deduplication (the KVBoost page's content hash, "Contexto"): sequences
that hold the same tokens share full pages after kvq_cache_dedup; a page that differs in one
token is not merged; decode reads exactly what it read before (bit for bit); a later write into a
shared page goes through copy-on-write and leaves the other sequences unchanged."""
import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, assert_close_attention


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (16, 16)])
def test_dedup_merges_identical_full_pages_only(kb, vb):
    m = kvq()
    H, D, G, P, layers = 2, 128, 4, 64, 2
    cache = m.Cache(n_layers=layers, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=5,
                    max_tokens=64 * 40, page_tokens=P)
    T = 300
    base = {l: (decode_kv(T, H, D, 10 + l), random_fp16((T, H, D), 20 + l)) for l in range(layers)}
    other = {l: (decode_kv(T, H, D, 30 + l), random_fp16((T, H, D), 40 + l)) for l in range(layers)}
    content = {}
    for l in range(layers):
        k, v = base[l]
        k3, v3 = k.clone(), v.clone()
        k3[150] = other[l][0][150]                                  # one token of page 2 differs
        content[l] = {0: (k, v), 1: (k, v),                         # sequence 1: same tokens as 0
                      2: (torch.cat([k[:128], other[l][0][128:]]), torch.cat([v[:128], other[l][1][128:]])),
                      3: (k3, v3),
                      4: other[l]}
    ids = [0, 1, 2, 3, 4]
    cache.extend(ids, [T] * 5)
    for l in range(layers):
        cache.append(l, ids, [T] * 5, torch.cat([content[l][s][0] for s in ids]).cuda(),
                     torch.cat([content[l][s][1] for s in ids]).cuda())
    q = random_fp16((5, H * G, D), 7).cuda()
    before = [cache.decode(l, ids, q) for l in range(layers)]
    mapped0 = cache.footprint()[1]
    freed = cache.dedup()
    cache.check()
    # full pages are 0..3 (positions 0..255): seq 1 shares all 4 with seq 0, seq 2 pages 0-1 with seq 0
    # and pages 2-3 with seq 4 (the same tokens), seq 3 pages 0, 1, 3 with seq 0
    assert freed == 4 + 2 + 2 + 3
    assert [cache.page(2, p) for p in (2, 3)] == [cache.page(4, p) for p in (2, 3)]
    page_bytes = mapped0 // (5 * 5)
    assert cache.footprint()[1] == mapped0 - freed * page_bytes
    assert [cache.page(1, p) for p in range(4)] == [cache.page(0, p) for p in range(4)]
    assert cache.page(3, 2) != cache.page(0, 2) and cache.page(3, 3) == cache.page(0, 3)
    assert cache.page(1, 4) != cache.page(0, 4)                    # partial pages are never merged
    for l in range(layers):
        assert torch.equal(cache.decode(l, ids, q), before[l]), f"layer {l}: reads changed"
    assert cache.dedup() == 0                                       # nothing left to merge
    # write into a shared page: truncate seq 1 into page 3 and append new tokens (copy-on-write)
    cache.truncate(1, 200)
    cache.extend([1], [10])
    new = {l: (decode_kv(10, H, D, 60 + l), random_fp16((10, H, D), 70 + l)) for l in range(layers)}
    for l in range(layers):
        cache.append(l, [1], [10], new[l][0].cuda(), new[l][1].cuda())
    cache.check()
    for l in range(layers):
        assert torch.equal(cache.decode(l, [0, 2, 3, 4], q[[0, 2, 3, 4]].contiguous()), before[l][[0, 2, 3, 4]])
        k = torch.cat([content[l][1][0][:200], new[l][0]])
        v = torch.cat([content[l][1][1][:200], new[l][1]])
        ref = oracle.attention_decode_batch(q[1:2].cpu().numpy(), [(oracle_dequant(k, kb), oracle_dequant(v, vb))])
        assert_close_attention(cache.decode(l, [1], q[1:2].contiguous()), ref, f"after copy-on-write, layer {l}")
    cache.close()
