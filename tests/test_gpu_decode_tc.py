"""GPU parity of the tensor-core decode kernel (cache flag
KVQ_CACHE_DECODE_TENSOR_CORES: scores as tcgen05 int8 MMAs on the stored key
codes, PV as fp16 MMAs) against the oracle's float64 softmax attention, on the
shapes it serves (8-bit keys, head_dim 128), and against the CUDA-core kernel
on the same cache contents."""
import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, assert_close_attention, ATOL, RTOL


def _build(m, kb, vb, H, lens, decode_tc, seed=0, page_tokens=256, layers=1):
    D = 128
    cache = m.Cache(n_layers=layers, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=len(lens) + 1,
                    max_tokens=sum(lens) + 256 * (len(lens) + 1), page_tokens=page_tokens, decode_tc=decode_tc)
    ids = list(range(len(lens)))
    cache.extend(ids, lens)
    hat = {}
    for layer in range(layers):
        ks = [decode_kv(L, H, D, seed + 100 * s + layer) for s, L in enumerate(lens)]
        vs = [random_fp16((L, H, D), seed + 7 + 100 * s + layer) for s, L in enumerate(lens)]
        cache.append(layer, ids, lens, torch.cat(ks).cuda(), torch.cat(vs).cuda())
        for s in ids:
            hat[(layer, s)] = (oracle_dequant(ks[s], kb), oracle_dequant(vs[s], vb))
    return cache, ids, hat


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (8, 8)])
@pytest.mark.parametrize("H,G", [(8, 4), (2, 2), (1, 8), (4, 1), (8, 8)])
def test_tc_decode_matches_oracle(kb, vb, H, G):
    m = kvq()
    lens = [1, 5, 127, 128, 129, 300, 1000, 2049]   # ragged tails around the 128-token tile
    cache, ids, hat = _build(m, kb, vb, H, lens, True, layers=2)
    for layer in range(2):
        q = random_fp16((len(lens), H * G, 128), 77 + layer)
        out = cache.decode(layer, ids, q.cuda())
        cache.check()
        ref = oracle.attention_decode_batch(q.numpy(), [hat[(layer, s)] for s in ids])
        assert_close_attention(out, ref, f"K{kb}V{vb} H{H} G{G} layer {layer}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (8, 8)])
def test_tc_decode_long_sequence_and_batch_mix(kb, vb):
    """Items split over many CTAs (combine kernel) next to short ones; same as the CUDA-core kernel."""
    m = kvq()
    H, G = 8, 4
    lens = [20011, 3, 700]
    tc, ids, hat = _build(m, kb, vb, H, lens, True, seed=5)
    cc, _, _ = _build(m, kb, vb, H, lens, False, seed=5)
    q = random_fp16((len(lens), H * G, 128), 5).cuda()
    out_tc = tc.decode(0, ids, q)
    out_cc = cc.decode(0, ids, q)
    tc.check()
    cc.check()
    ref = oracle.attention_decode_batch(q.cpu().numpy(), [hat[(0, s)] for s in ids])
    assert_close_attention(out_tc, ref, "tc")
    assert_close_attention(out_cc, ref, "cuda cores")
    assert torch.allclose(out_tc.float(), out_cc.float(), atol=2 * ATOL, rtol=2 * RTOL)
    tc.close()
    cc.close()


@pytest.mark.gpu
@pytest.mark.parametrize("page_tokens", [64, 192, 320])
def test_tc_decode_small_pages_and_scale(page_tokens):
    """Pages that are not a multiple of the 128-token tile: chunks of 64 tokens, rows past the page zero-filled."""
    m = kvq()
    H, G = 2, 4
    lens = [65, 200, 1, 700]
    cache, ids, hat = _build(m, 8, 4, H, lens, True, page_tokens=page_tokens)
    q = random_fp16((len(lens), H * G, 128), 11)
    out = cache.decode(0, ids, q.cuda(), softmax_scale=0.05)
    cache.check()
    ref = oracle.attention_decode_batch(q.numpy(), [hat[(0, s)] for s in ids], scale=0.05)
    assert_close_attention(out, ref, f"page {page_tokens}")
    cache.close()


@pytest.mark.gpu
def test_tc_decode_after_incremental_appends():
    m = kvq()
    H, G, D = 2, 4, 128
    cache = m.Cache(1, H, D, 8, 4, max_seqs=2, max_tokens=4096, decode_tc=True)
    ks, vs = [], []
    for step in range(260):
        cache.extend([0], [1])
        k = decode_kv(1, H, D, 300 + step)
        v = random_fp16((1, H, D), 900 + step)
        cache.append(0, [0], [1], k.cuda(), v.cuda())
        ks.append(k)
        vs.append(v)
        if step in (0, 1, 127, 128, 255, 256, 259):
            q = random_fp16((1, H * G, D), step)
            out = cache.decode(0, [0], q.cuda())
            ref = oracle.attention_decode(q[0].numpy(), oracle_dequant(torch.cat(ks), 8),
                                          oracle_dequant(torch.cat(vs), 4))[None]
            assert_close_attention(out, ref, f"step {step}")
    cache.check()
    cache.close()
