"""GPU parity: split-KV decode attention against the oracle's float64 softmax
attention over its own dequantisation of the same fp16 inputs."""

import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, assert_close_attention

FORMATS = [(8, 4), (8, 8), (4, 4), (4, 8), (16, 16)]


def _build(m, kb, vb, D, H, lens, layers=1, seed=0, page_tokens=256):
    cache = m.Cache(n_layers=layers, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=len(lens) + 1,
                    max_tokens=sum(lens) + 256 * (len(lens) + 1), page_tokens=page_tokens)
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
@pytest.mark.parametrize("kb,vb", FORMATS)
@pytest.mark.parametrize("D,H,G", [(64, 4, 8), (128, 8, 4), (128, 2, 2), (64, 2, 1), (128, 1, 8)])
def test_decode_matches_oracle(kb, vb, D, H, G):
    m = kvq()
    lens = [1, 5, 32, 129, 300, 1000]
    cache, ids, hat = _build(m, kb, vb, D, H, lens, layers=2)
    for layer in range(2):
        q = random_fp16((len(lens), H * G, D), 77 + layer)
        out = cache.decode(layer, ids, q.cuda())
        cache.check()
        ref = oracle.attention_decode_batch(q.numpy(), [hat[(layer, s)] for s in ids])
        assert_close_attention(out, ref, f"K{kb}V{vb} D{D} H{H} G{G} layer {layer}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (8, 8), (4, 4), (4, 8)])
@pytest.mark.parametrize("D,G", [(128, 4), (128, 8), (64, 8), (64, 1)])
def test_decode_256_token_stages(kb, vb, D, G):
    """A step with at least two 256-token chunks per CTA on 256-token pages runs the kernel with
    256-token stages (128-token ones where three of them do not fit, K8V8 at head_dim 128); the
    second sequence ends in a ragged chunk."""
    m = kvq()
    H = 8
    lens = [10000, 300]
    cache, ids, hat = _build(m, kb, vb, D, H, lens)
    q = random_fp16((len(lens), H * G, D), 11 + G)
    out = cache.decode(0, ids, q.cuda())
    cache.check()
    ref = oracle.attention_decode_batch(q.numpy(), [hat[(0, s)] for s in ids])
    assert_close_attention(out, ref, f"K{kb}V{vb} D{D} G{G}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("page_tokens", [512, 768])
def test_decode_256_token_stages_in_larger_pages(page_tokens):
    """256-token chunks at offsets 0, 256 (and 512) inside one page."""
    m = kvq()
    D, H, G = 128, 8, 4
    lens = [10000, 700]
    cache, ids, hat = _build(m, 8, 4, D, H, lens, page_tokens=page_tokens)
    q = random_fp16((len(lens), H * G, D), 21)
    out = cache.decode(0, ids, q.cuda())
    cache.check()
    ref = oracle.attention_decode_batch(q.numpy(), [hat[(0, s)] for s in ids])
    assert_close_attention(out, ref, f"pages of {page_tokens}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (16, 16)])
def test_decode_long_sequence_spans_many_ctas(kb, vb):
    """One long sequence: every item is split over many CTAs and merged by the combine kernel."""
    m = kvq()
    D, H, G = 128, 8, 4
    lens = [20011]
    cache, ids, hat = _build(m, kb, vb, D, H, lens)
    q = random_fp16((1, H * G, D), 5)
    out = cache.decode(0, ids, q.cuda())
    cache.check()
    ref = oracle.attention_decode_batch(q.numpy(), [hat[(0, 0)]])
    assert_close_attention(out, ref, "long")
    cache.close()


@pytest.mark.gpu
def test_decode_is_independent_of_batch_composition():
    m = kvq()
    D, H, G = 128, 8, 4
    lens = [700, 3000, 45, 1]
    cache, ids, hat = _build(m, 8, 4, D, H, lens)
    q = random_fp16((len(lens), H * G, D), 9).cuda()
    full = cache.decode(0, ids, q)
    for i in ids:
        one = cache.decode(0, [i], q[i:i + 1].contiguous())
        assert torch.allclose(one.float(), full[i:i + 1].float(), atol=2e-3, rtol=1e-2)
    rev = cache.decode(0, ids[::-1], q.flip(0).contiguous())
    assert torch.allclose(rev.flip(0).float(), full.float(), atol=2e-3, rtol=1e-2)
    cache.check()
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("page_tokens,D", [(64, 64), (192, 64), (64, 128), (320, 128)])
def test_decode_softmax_scale_and_small_pages(page_tokens, D):
    """Pages smaller than (or not a multiple of) the kernel's stage: work chunks must stay inside a page."""
    m = kvq()
    H, G = 2, 4
    lens = [65, 200, 1, 700]
    cache, ids, hat = _build(m, 8, 4, D, H, lens, page_tokens=page_tokens)
    q = random_fp16((len(lens), H * G, D), 11)
    out = cache.decode(0, ids, q.cuda(), softmax_scale=0.05)
    cache.check()
    ref = oracle.attention_decode_batch(q.numpy(), [hat[(0, s)] for s in ids], scale=0.05)
    assert_close_attention(out, ref, "scale 0.05")
    cache.close()


@pytest.mark.gpu
def test_decode_after_incremental_appends():
    """Decode step by step while tokens are appended one at a time (the serving loop)."""
    m = kvq()
    D, H, G = 128, 2, 4
    cache = m.Cache(1, H, D, 8, 4, max_seqs=2, max_tokens=4096)
    ks, vs = [], []
    for step in range(300):
        cache.extend([0], [1])
        k = decode_kv(1, H, D, 300 + step)
        v = random_fp16((1, H, D), 900 + step)
        cache.append(0, [0], [1], k.cuda(), v.cuda())
        ks.append(k)
        vs.append(v)
        if step in (0, 1, 31, 32, 255, 256, 299):
            q = random_fp16((1, H * G, D), step)
            out = cache.decode(0, [0], q.cuda())
            kh = oracle_dequant(torch.cat(ks), 8)
            vh = oracle_dequant(torch.cat(vs), 4)
            ref = oracle.attention_decode(q[0].numpy(), kh, vh)[None]
            assert_close_attention(out, ref, f"step {step}")
    cache.check()
    cache.close()


@pytest.mark.gpu
def test_decode_step_replays_from_a_cuda_graph():
    """One decode step through the API (extend, then append + decode for every layer) captured in a CUDA
    graph and replayed: each replay re-appends the same token and gives the eager result bit for bit,
    within tolerance of the oracle.  Sequence 0 crosses a page boundary inside the captured step."""
    m = kvq()
    D, H, G, layers = 128, 8, 4, 2
    lens = [256, 700]
    B = len(lens)
    cache, ids, hat = _build(m, 8, 4, D, H, lens, layers=layers)
    k_new = [decode_kv(B, H, D, 500 + l) for l in range(layers)]
    v_new = [random_fp16((B, H, D), 600 + l) for l in range(layers)]
    q = [random_fp16((B, H * G, D), 700 + l) for l in range(layers)]
    kd, vd, qd = [t.cuda() for t in k_new], [t.cuda() for t in v_new], [t.cuda() for t in q]
    out = [torch.empty_like(t) for t in qd]
    ws = torch.empty(cache.decode_workspace_size(B, H * G), dtype=torch.uint8, device="cuda")
    cache.decode(0, ids, qd[0], out=out[0], workspace=ws)      # first-call setup outside the capture
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cache.extend(ids, [1] * B)
        for layer in range(layers):
            cache.append(layer, ids, [1] * B, kd[layer], vd[layer])
            cache.decode(layer, ids, qd[layer], out=out[layer], workspace=ws)
    assert [cache.length(s) for s in ids] == [n + 1 for n in lens]
    for o in out:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    first = [o.clone() for o in out]
    g.replay()
    torch.cuda.synchronize()
    cache.check()
    for layer in range(layers):
        assert torch.equal(out[layer], first[layer]), f"layer {layer}: replays differ"
        eager = cache.decode(layer, ids, qd[layer])
        assert torch.equal(eager, first[layer]), f"layer {layer}: replay differs from the eager call"
        kv = []
        for s in ids:
            kh, vh = hat[(layer, s)]
            kh = np.concatenate([kh, oracle_dequant(k_new[layer][s:s + 1], 8)])
            vh = np.concatenate([vh, oracle_dequant(v_new[layer][s:s + 1], 4)])
            kv.append((kh, vh))
        ref = oracle.attention_decode_batch(q[layer].numpy(), kv)
        assert_close_attention(first[layer], ref, f"graph replay layer {layer}")
    del g
    cache.close()


@pytest.mark.gpu
def test_decode_at_the_maximum_batch():
    """KVQ_MAX_BATCH sequences in one call (the batch descriptors travel as kernel parameters), with
    lengths from 1 to a few pages; every output checked against the oracle."""
    m = kvq()
    D, H, G = 64, 2, 4
    B = m.KVQ_MAX_BATCH
    rng = np.random.default_rng(11)
    lens = [int(x) for x in rng.integers(1, 700, size=B)]
    lens[0], lens[-1] = 1, 256
    cache, ids, hat = _build(m, 8, 4, D, H, lens)
    q = random_fp16((B, H * G, D), 21)
    out = cache.decode(0, ids, q.cuda())
    cache.check()
    ref = oracle.attention_decode_batch(q.numpy(), [hat[(0, s)] for s in ids])
    assert_close_attention(out, ref, "max batch")
    cache.close()


@pytest.mark.gpu
def test_fork_shares_a_prefix_and_copies_on_write():
    """kvq_seq_fork: two sequences started from one cached prefix read the same pages; new tokens appended
    to each afterwards (the shared, partly filled last page is copied first) leave the other intact."""
    m = kvq()
    D, H, G, layers = 128, 2, 4, 2
    T = 300
    cache = m.Cache(n_layers=layers, n_kv_heads=H, head_dim=D, k_bits=8, v_bits=4, max_seqs=4, max_tokens=4096)
    cache.extend([0], [T])
    base = {}
    for layer in range(layers):
        k = decode_kv(T, H, D, 40 + layer)
        v = random_fp16((T, H, D), 50 + layer)
        cache.append(layer, [0], [T], k.cuda(), v.cuda())
        base[layer] = (k, v)
    cache.fork(0, 1)                 # all 300 positions
    cache.fork(0, 2, 200)            # a prefix ending inside the first page
    assert cache.page(1, 1) == cache.page(0, 1) and cache.page(2, 0) == cache.page(0, 0)
    q = [random_fp16((3, H * G, D), 60 + layer) for layer in range(layers)]
    same = cache.decode(0, [0, 1], q[0][:1].repeat(2, 1, 1).cuda())     # one query for both sequences
    assert torch.equal(same[0], same[1])
    cache.extend([0, 1, 2], [1, 1, 1])
    assert cache.page(0, 1) != cache.page(1, 1) and cache.page(2, 0) != cache.page(0, 0)
    new = {}
    for layer in range(layers):
        k = decode_kv(3, H, D, 70 + layer)
        v = random_fp16((3, H, D), 80 + layer)
        cache.append(layer, [0, 1, 2], [1, 1, 1], k.cuda(), v.cuda())
        new[layer] = (k, v)
    cache.check()
    prefix = {0: T, 1: T, 2: 200}
    for layer in range(layers):
        out = cache.decode(layer, [0, 1, 2], q[layer].cuda())
        kv = []
        for s in range(3):
            k = torch.cat([base[layer][0][:prefix[s]], new[layer][0][s:s + 1]])
            v = torch.cat([base[layer][1][:prefix[s]], new[layer][1][s:s + 1]])
            kv.append((oracle_dequant(k, 8), oracle_dequant(v, 4)))
        ref = oracle.attention_decode_batch(q[layer].numpy(), kv)
        assert_close_attention(out, ref, f"fork layer {layer}")
    cache.release(0)
    cache.release(2)
    out1 = cache.decode(0, [1], q[0][1:2].cuda())       # seq 1 still reads its pages
    k = torch.cat([base[0][0], new[0][0][1:2]])
    v = torch.cat([base[0][1], new[0][1][1:2]])
    ref = oracle.attention_decode_batch(q[0][1:2].numpy(), [(oracle_dequant(k, 8), oracle_dequant(v, 4))])
    assert_close_attention(out1, ref, "fork after release")
    cache.check()
    cache.close()
