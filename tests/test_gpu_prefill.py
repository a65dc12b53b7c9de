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


@pytest.mark.gpu
def test_prefill_in_bounded_waves_matches_oracle_and_replays():
    """A batch whose dequantised tiles exceed one wave: the long sequence is split into KV-head ranges,
    the short ones form a wave of their own; waves alternate between two internal streams and two
    halves of a bounded workspace (smaller than the whole cache in fp16).  Every row matches the oracle,
    and a CUDA graph of the call (fork / join of the internal streams) replays it bit for bit."""
    m = kvq()
    kb, vb, D, H, G = 8, 4, 128, 8, 4
    cached, chunk = [13000, 3000, 100], [64, 129, 1]
    n = len(cached)
    cache = m.Cache(n_layers=1, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=n,
                    max_tokens=sum(cached) + sum(chunk) + 256 * n)
    ids = list(range(n))
    ks = [decode_kv(c + q, H, D, 300 + s) for s, (c, q) in enumerate(zip(cached, chunk))]
    vs = [random_fp16((c + q, H, D), 400 + s) for s, (c, q) in enumerate(zip(cached, chunk))]
    cache.extend(ids, [c + q for c, q in zip(cached, chunk)])
    cache.append(0, ids, [c + q for c, q in zip(cached, chunk)], torch.cat(ks).cuda(), torch.cat(vs).cuda())
    ws_need = cache.prefill_workspace_size(ids, chunk, H * G)
    whole = sum(-(-(c + q) // 64) for c, q in zip(cached, chunk)) * H * 64 * D * 3 * 2
    assert ws_need < whole                                    # bounded: not the whole cache in fp16
    q = random_fp16((sum(chunk), H * G, D), 77).cuda()
    out = cache.prefill(0, ids, chunk, q)
    cache.check()
    off = 0
    for s in ids:
        ref = oracle.attention_prefill(q[off: off + chunk[s]].cpu().numpy(), oracle_dequant(ks[s], kb),
                                       oracle_dequant(vs[s], vb), cached[s])
        assert_close_attention(out[off: off + chunk[s]], ref, f"wave prefill seq {s}")
        off += chunk[s]
    ws = torch.empty(ws_need, dtype=torch.uint8, device="cuda")
    out2 = torch.empty_like(q)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cache.prefill(0, ids, chunk, q, out=out2, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    cache.check()
    assert torch.equal(out2, out)
    del g
    cache.close()
