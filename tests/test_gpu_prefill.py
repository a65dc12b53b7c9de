"""GPU parity: chunked prefill (tcgen05) against the oracle's causal float64
attention over its own dequantisation of the same fp16 inputs.  The kernel
rounds the dequantised K / V and the probabilities to fp16 before the tensor
cores (fp32 accumulation); the tolerance is the suite's."""
import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, assert_close_attention


def _run(m, kb, vb, D, H, G, cached, chunk, seed=0, page_tokens=256):
    n = len(cached)
    cache = m.Cache(n_layers=1, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=n,
                    max_tokens=sum(cached) + sum(chunk) + 256 * n, page_tokens=page_tokens)
    ids = list(range(n))
    ks = [decode_kv(c + q, H, D, seed + 10 * s) for s, (c, q) in enumerate(zip(cached, chunk))]
    vs = [random_fp16((c + q, H, D), seed + 5 + 10 * s) for s, (c, q) in enumerate(zip(cached, chunk))]
    # the cached part first (as an earlier prefill would), then the chunk
    pre = [s for s in ids if cached[s] > 0]
    if pre:
        cache.extend(pre, [cached[s] for s in pre])
        cache.append(0, pre, [cached[s] for s in pre], torch.cat([ks[s][:cached[s]] for s in pre]).cuda(),
                     torch.cat([vs[s][:cached[s]] for s in pre]).cuda())
    cache.extend(ids, chunk)
    cache.append(0, ids, chunk, torch.cat([ks[s][cached[s]:] for s in ids]).cuda(),
                 torch.cat([vs[s][cached[s]:] for s in ids]).cuda())
    q = random_fp16((sum(chunk), H * G, D), seed + 99)
    out = cache.prefill(0, ids, chunk, q.cuda())
    cache.check()
    off = 0
    for s in ids:
        kh, vh = oracle_dequant(ks[s], kb), oracle_dequant(vs[s], vb)
        ref = oracle.attention_prefill(q[off: off + chunk[s]].numpy(), kh, vh, cached[s])
        assert_close_attention(out[off: off + chunk[s]], ref, f"seq {s} cached {cached[s]} chunk {chunk[s]}")
        off += chunk[s]
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (16, 16), (8, 8), (4, 4), (4, 8)])
@pytest.mark.parametrize("D", [64, 128])
def test_prefill_matches_oracle_ragged(kb, vb, D):
    m = kvq()
    _run(m, kb, vb, D=D, H=2, G=4, cached=[0, 100, 300, 129], chunk=[64, 200, 129, 1])


@pytest.mark.gpu
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_prefill_gqa_and_head_dims(G, D):
    m = kvq()
    _run(m, 8, 4, D=D, H=2, G=G, cached=[37, 0], chunk=[150, 70], seed=G * 7 + D)


@pytest.mark.gpu
def test_prefill_long_cache_many_tiles():
    m = kvq()
    _run(m, 8, 4, D=128, H=1, G=4, cached=[3000], chunk=[333], seed=3)


@pytest.mark.gpu
def test_prefill_small_pages():
    m = kvq()
    _run(m, 8, 4, D=128, H=2, G=4, cached=[65, 190], chunk=[100, 67], seed=4, page_tokens=64)


@pytest.mark.gpu
def test_prefill_rows_agree_with_decode():
    """A one-row chunk is a decode step: the two kernels must agree."""
    m = kvq()
    D, H, G = 128, 2, 4
    cache = m.Cache(1, H, D, 8, 4, max_seqs=1, max_tokens=2048)
    cache.extend([0], [1000])
    cache.append(0, [0], [1000], decode_kv(1000, H, D, 1).cuda(), random_fp16((1000, H, D), 2).cuda())
    q = random_fp16((1, H * G, D), 3).cuda()
    a = cache.prefill(0, [0], [1], q)
    b = cache.decode(0, [0], q.view(1, H * G, D))
    cache.check()
    assert torch.allclose(a.float(), b.float(), atol=2e-3, rtol=1e-2)
    cache.close()
