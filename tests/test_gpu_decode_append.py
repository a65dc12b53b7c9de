"""GPU parity of kvq_decode_append_attn, the one-token decode step: the new token's K / V are
quantised into position len - 1 (codes and scales bit-exact against the oracle's quantiser) and the
query attends to positions 0 .. len - 1 (within tolerance of the oracle's float64 attention).  For
quantized caches the append is fused into the decode kernel; its result must equal, bit for bit, the
separate kvq_append + kvq_decode_attn calls."""

import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, oracle_export, assert_close_attention

FORMATS = [(8, 4), (8, 8), (4, 4), (4, 8), (16, 16)]


def _fill(m, kb, vb, D, H, lens, layers=1, seed=0, page_tokens=256, extra=64):
    cache = m.Cache(n_layers=layers, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=len(lens) + 1,
                    max_tokens=sum(lens) + (256 + extra) * (len(lens) + 1), page_tokens=page_tokens)
    ids = list(range(len(lens)))
    cache.extend(ids, lens)
    raw = {}
    for layer in range(layers):
        ks = [decode_kv(L, H, D, seed + 100 * s + layer) for s, L in enumerate(lens)]
        vs = [random_fp16((L, H, D), seed + 7 + 100 * s + layer) for s, L in enumerate(lens)]
        cache.append(layer, ids, lens, torch.cat(ks).cuda(), torch.cat(vs).cuda())
        for s in ids:
            raw[(layer, s)] = (ks[s], vs[s])
    return cache, ids, raw


def _check_row(cache, layer, s, pos, k, v, kb, vb):
    exp = cache.export(layer, s, pos, 1)
    for name, x, bits in (("k", k, kb), ("v", v, vb)):
        codes, scales = oracle_export(x, bits)
        got = exp[f"{name}_codes"].cpu().numpy()
        if bits == 16:
            assert (got.view(np.uint16) == codes.view(np.uint16)).all(), f"{name} fp16 copy differs"
        else:
            assert (got == codes).all(), f"{name} codes differ from the oracle"
            assert (exp[f"{name}_scales"].cpu().numpy().view(np.uint16) == scales.view(np.uint16)).all(), \
                f"{name} scales differ from the oracle"


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", FORMATS)
@pytest.mark.parametrize("D,H,G", [(128, 8, 4), (64, 4, 8), (128, 2, 1), (64, 2, 2)])
def test_decode_append_matches_oracle_and_the_separate_calls(kb, vb, D, H, G):
    m = kvq()
    lens = [1, 127, 128, 300, 2000]           # the new token lands at the start, inside and at the end of a chunk
    cache, ids, raw = _fill(m, kb, vb, D, H, lens)
    twin, _, _ = _fill(m, kb, vb, D, H, lens)
    B = len(lens)
    k_new = decode_kv(B, H, D, 4242)
    v_new = random_fp16((B, H, D), 4343)
    q = random_fp16((B, H * G, D), 4444)
    cache.extend(ids, [1] * B)
    out = cache.decode_append(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    twin.extend(ids, [1] * B)
    twin.append(0, ids, [1] * B, k_new.cuda(), v_new.cuda())
    sep = twin.decode(0, ids, q.cuda())
    twin.check()
    assert torch.equal(out, sep), "fused step differs from append + decode"
    kv = []
    for s in ids:
        _check_row(cache, 0, s, lens[s], k_new[s:s + 1], v_new[s:s + 1], kb, vb)
        k = torch.cat([raw[(0, s)][0], k_new[s:s + 1]])
        v = torch.cat([raw[(0, s)][1], v_new[s:s + 1]])
        kv.append((oracle_dequant(k, kb), oracle_dequant(v, vb)))
    ref = oracle.attention_decode_batch(q.numpy(), kv)
    assert_close_attention(out, ref, f"K{kb}V{vb} D{D} G{G}")
    cache.close()
    twin.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (4, 4), (4, 8), (8, 8)])
@pytest.mark.parametrize("D,G", [(128, 4), (64, 8)])
def test_decode_append_256_token_stages(kb, vb, D, G):
    """A step large enough for 256-token stages (at least two 256-token chunks per CTA): the new token
    lands at the start, inside and at the end of a 256-token chunk; the fused step equals the separate
    calls bit for bit and the oracle within tolerance, and the appended row is bit-exact."""
    m = kvq()
    H = 8
    lens = [10000, 255, 256, 511]
    cache, ids, raw = _fill(m, kb, vb, D, H, lens)
    twin, _, _ = _fill(m, kb, vb, D, H, lens)
    B = len(lens)
    k_new = decode_kv(B, H, D, 5252)
    v_new = random_fp16((B, H, D), 5353)
    q = random_fp16((B, H * G, D), 5454)
    cache.extend(ids, [1] * B)
    out = cache.decode_append(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    twin.extend(ids, [1] * B)
    twin.append(0, ids, [1] * B, k_new.cuda(), v_new.cuda())
    sep = twin.decode(0, ids, q.cuda())
    twin.check()
    assert torch.equal(out, sep), "fused step differs from append + decode"
    kv = []
    for s in ids:
        _check_row(cache, 0, s, lens[s], k_new[s:s + 1], v_new[s:s + 1], kb, vb)
        k = torch.cat([raw[(0, s)][0], k_new[s:s + 1]])
        v = torch.cat([raw[(0, s)][1], v_new[s:s + 1]])
        kv.append((oracle_dequant(k, kb), oracle_dequant(v, vb)))
    assert_close_attention(out, oracle.attention_decode_batch(q.numpy(), kv), f"K{kb}V{vb} D{D} G{G}")
    cache.close()
    twin.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (4, 8)])
def test_decode_append_serving_loop_across_pages(kb, vb):
    """300 one-token steps on two layers with 64-token pages: every step's output against the oracle at a
    few steps, and every appended row bit-exact at the end."""
    m = kvq()
    D, H, G, layers = 128, 2, 4, 2
    cache = m.Cache(layers, H, D, kb, vb, max_seqs=2, max_tokens=4096, page_tokens=64)
    ks = {l: [] for l in range(layers)}
    vs = {l: [] for l in range(layers)}
    for step in range(300):
        cache.extend([0, 1], [1, 1])
        for layer in range(layers):
            k = decode_kv(2, H, D, 1000 * layer + step)
            v = random_fp16((2, H, D), 5000 + 1000 * layer + step)
            q = random_fp16((2, H * G, D), 9000 + 1000 * layer + step)
            out = cache.decode_append(layer, [0, 1], q.cuda(), k.cuda(), v.cuda())
            ks[layer].append(k)
            vs[layer].append(v)
            if step in (0, 1, 63, 64, 200, 299):
                kv = []
                for s in range(2):
                    kk = torch.stack([x[s] for x in ks[layer]])
                    vv = torch.stack([x[s] for x in vs[layer]])
                    kv.append((oracle_dequant(kk, kb), oracle_dequant(vv, vb)))
                ref = oracle.attention_decode_batch(q.numpy(), kv)
                assert_close_attention(out, ref, f"step {step} layer {layer}")
    cache.check()
    for layer in range(layers):
        for s in range(2):
            exp = cache.export(layer, s, 0, 300)
            kc, ksc = oracle_export(torch.stack([x[s] for x in ks[layer]]), kb)
            assert (exp["k_codes"].cpu().numpy() == kc).all()
            assert (exp["k_scales"].cpu().numpy().view(np.uint16) == ksc.view(np.uint16)).all()
    cache.close()


@pytest.mark.gpu
def test_decode_append_step_replays_from_a_cuda_graph():
    """The whole one-token step (extend, then one fused launch per layer) captured once and replayed:
    each replay re-appends the same token and matches the eager call bit for bit."""
    m = kvq()
    D, H, G, layers = 64, 4, 8, 3
    lens = [128, 1000, 5]
    B = len(lens)
    cache, ids, raw = _fill(m, 8, 4, D, H, lens, layers=layers)
    k_new = [decode_kv(B, H, D, 70 + l).cuda() for l in range(layers)]
    v_new = [random_fp16((B, H, D), 80 + l).cuda() for l in range(layers)]
    q = [random_fp16((B, H * G, D), 90 + l).cuda() for l in range(layers)]
    out = [torch.empty_like(t) for t in q]
    ws = torch.empty(cache.decode_workspace_size(B, H * G), dtype=torch.uint8, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cache.extend(ids, [1] * B)
        for layer in range(layers):
            cache.decode_append(layer, ids, q[layer], k_new[layer], v_new[layer], out=out[layer], workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    first = [o.clone() for o in out]
    g.replay()
    torch.cuda.synchronize()
    cache.check()
    for layer in range(layers):
        assert torch.equal(out[layer], first[layer])
        assert torch.equal(cache.decode(layer, ids, q[layer]), first[layer])
        kv = []
        for s in ids:
            k = torch.cat([raw[(layer, s)][0], k_new[layer][s:s + 1].cpu()])
            v = torch.cat([raw[(layer, s)][1], v_new[layer][s:s + 1].cpu()])
            kv.append((oracle_dequant(k, 8), oracle_dequant(v, 4)))
        assert_close_attention(first[layer], oracle.attention_decode_batch(q[layer].cpu().numpy(), kv),
                               f"replay layer {layer}")
    del g
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("G,H", [(8, 8), (4, 8)])
def test_decode_long_items_merged_by_the_last_cta_are_deterministic(G, H):
    """Items spread over many CTAs (one 70B-shaped sequence of 60000 tokens: every KV head spans ~18 CTAs)
    are merged inside the kernel by the last CTA to finish; the merge order is fixed, so two calls agree
    bit for bit, and both match the oracle."""
    m = kvq()
    D = 128
    lens = [60000]
    cache, ids, raw = _fill(m, 8, 4, D, H, lens)
    q = random_fp16((1, H * G, D), 31).cuda()
    a = cache.decode(0, ids, q)
    b = cache.decode(0, ids, q)
    cache.check()
    assert torch.equal(a, b)
    kv = [(oracle_dequant(raw[(0, 0)][0], 8), oracle_dequant(raw[(0, 0)][1], 4))]
    assert_close_attention(a, oracle.attention_decode_batch(q.cpu().numpy(), kv), f"G{G} 60000 tokens")
    cache.close()
