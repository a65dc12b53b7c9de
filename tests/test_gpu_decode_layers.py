"""GPU parity of kvq_decode_attn_layers, the layer-batched decode step: one launch per run of
consecutive same-format layers takes every (layer, sequence, KV head, slice) of the run.  The
appended rows are bit-exact against the oracle's quantiser (and equal to the per-layer calls'),
and every layer's output matches the oracle's float64 attention over that layer's dequantised
cache; runs split by format (per-layer precision) and by batch capacity, the rotating window,
256-token stages and graph replay are covered."""

import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, oracle_export, assert_close_attention

FORMATS = [(8, 4), (8, 8), (4, 4), (4, 8), (16, 16)]


def _fill(m, layer_bits, D, H, lens, seed=0, page_tokens=256, extra=64):
    kb, vb = layer_bits[0]
    cache = m.Cache(n_layers=len(layer_bits), n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb,
                    max_seqs=len(lens) + 1, max_tokens=(sum(lens) + (256 + extra) * (len(lens) + 1)),
                    page_tokens=page_tokens, layer_bits=layer_bits)
    ids = list(range(len(lens)))
    cache.extend(ids, lens)
    raw = {}
    for layer in range(len(layer_bits)):
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
            assert (got.view(np.uint16) == codes.view(np.uint16)).all(), f"layer {layer} {name} fp16 copy differs"
        else:
            assert (got == codes).all(), f"layer {layer} {name} codes differ from the oracle"
            assert (exp[f"{name}_scales"].cpu().numpy().view(np.uint16) == scales.view(np.uint16)).all(), \
                f"layer {layer} {name} scales differ from the oracle"


def _step_inputs(NL, B, H, G, D, seed):
    k_new = torch.stack([decode_kv(B, H, D, seed + l) for l in range(NL)])
    v_new = torch.stack([random_fp16((B, H, D), seed + 100 + l) for l in range(NL)])
    q = torch.stack([random_fp16((B, H * G, D), seed + 200 + l) for l in range(NL)])
    return q, k_new, v_new


def _reference(q_l, raw, layer, ids, kb, vb, k_new=None, v_new=None):
    kv = []
    for s in ids:
        k, v = raw[(layer, s)]
        if k_new is not None:
            k = torch.cat([k, k_new[s:s + 1]])
            v = torch.cat([v, v_new[s:s + 1]])
        kv.append((oracle_dequant(k, kb), oracle_dequant(v, vb)))
    return oracle.attention_decode_batch(q_l.numpy(), kv)


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", FORMATS)
@pytest.mark.parametrize("D,H,G", [(128, 8, 4), (64, 4, 8)])
def test_layer_batched_step_matches_oracle_and_per_layer_calls(kb, vb, D, H, G):
    m = kvq()
    NL = 3
    lens = [1, 127, 300, 2000]                # the new token at the start, inside and at the end of a chunk
    cache, ids, raw = _fill(m, [(kb, vb)] * NL, D, H, lens)
    twin, _, _ = _fill(m, [(kb, vb)] * NL, D, H, lens)
    B = len(lens)
    q, k_new, v_new = _step_inputs(NL, B, H, G, D, 300)
    cache.extend(ids, [1] * B)
    out = cache.decode_layers(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    twin.extend(ids, [1] * B)
    sep = torch.stack([twin.decode_append(l, ids, q[l].cuda(), k_new[l].cuda(), v_new[l].cuda()) for l in range(NL)])
    twin.check()
    for l in range(NL):
        for s in ids:
            _check_row(cache, l, s, lens[s], k_new[l, s:s + 1], v_new[l, s:s + 1], kb, vb)
            a = cache.export(l, s, lens[s], 1)
            b = twin.export(l, s, lens[s], 1)
            for key in a:
                if a[key] is None:                    # fp16 layers have no scales
                    assert b[key] is None
                else:
                    assert torch.equal(a[key], b[key]), f"layer {l} seq {s} {key}: batched and per-layer rows differ"
        ref = _reference(q[l], raw, l, ids, kb, vb, k_new[l], v_new[l])
        assert_close_attention(out[l], ref, f"layer {l} K{kb}V{vb} D{D} G{G}")
        assert_close_attention(sep[l], ref, f"per-layer call, layer {l}")
    cache.close()
    twin.close()


@pytest.mark.gpu
@pytest.mark.parametrize("D,H,G", [(128, 2, 4), (64, 4, 8)])
def test_layer_batched_step_over_mixed_precision_layers(D, H, G):
    """Layers of five formats: the call splits into one launch per format run; a sub-range of layers
    (layer0 = 1) reads and writes only its own layers."""
    m = kvq()
    layer_bits = [(8, 4), (8, 4), (4, 8), (16, 16), (16, 16), (8, 8), (4, 4)]
    NL = len(layer_bits)
    lens = [300, 37, 1000]
    cache, ids, raw = _fill(m, layer_bits, D, H, lens, seed=11)
    B = len(lens)
    # decode only (no append) over every layer
    q, _, _ = _step_inputs(NL, B, H, G, D, 900)
    out = cache.decode_layers(0, ids, q.cuda())
    cache.check()
    for l, (kb, vb) in enumerate(layer_bits):
        assert_close_attention(out[l], _reference(q[l], raw, l, ids, kb, vb), f"decode layer {l} K{kb}V{vb}")
    # one appending step over layers 1 .. 5
    cache.extend(ids, [1] * B)
    q, k_new, v_new = _step_inputs(5, B, H, G, D, 1900)
    before0 = cache.export(0, 0, lens[0], 1)
    before6 = cache.export(6, 0, lens[0], 1)
    out = cache.decode_layers(1, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    for i in range(5):
        l = 1 + i
        kb, vb = layer_bits[l]
        for s in ids:
            _check_row(cache, l, s, lens[s], k_new[i, s:s + 1], v_new[i, s:s + 1], kb, vb)
        ref = _reference(q[i], raw, l, ids, kb, vb, k_new[i], v_new[i])
        assert_close_attention(out[i], ref, f"step layer {l} K{kb}V{vb}")
    for l, before in ((0, before0), (6, before6)):
        after = cache.export(l, 0, lens[0], 1)
        for key in before:
            if before[key] is not None:
                assert torch.equal(before[key], after[key]), f"layer {l} outside the call was written"
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (16, 16)])
def test_layer_batched_step_split_by_batch_capacity(kb, vb):
    """100 sequences x 3 layers exceed one batch (256 entries): two layers go to the first launch and
    one to the second, reusing the workspace in stream order."""
    m = kvq()
    D, H, G, NL = 64, 2, 4, 3
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1, 200, size=100)]
    cache, ids, raw = _fill(m, [(kb, vb)] * NL, D, H, lens, seed=21, page_tokens=64, extra=0)
    B = len(lens)
    assert cache.decode_layers_workspace_size(NL, B, H * G) == cache.decode_workspace_size(2 * B, H * G)
    q, k_new, v_new = _step_inputs(NL, B, H, G, D, 2900)
    cache.extend(ids, [1] * B)
    out = cache.decode_layers(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    for l in range(NL):
        for s in (0, 17, 99):
            _check_row(cache, l, s, lens[s], k_new[l, s:s + 1], v_new[l, s:s + 1], kb, vb)
        ref = _reference(q[l], raw, l, ids, kb, vb, k_new[l], v_new[l])
        assert_close_attention(out[l], ref, f"layer {l}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (4, 4)])
def test_layer_batched_step_256_token_stages(kb, vb):
    """Four layers of two long sequences: the batched step has enough 256-token chunks for 256-token
    stages (a single layer of it does not), and its CTA ranges cross layer boundaries."""
    m = kvq()
    D, H, G, NL = 128, 8, 4, 4
    lens = [3000, 5000]
    cache, ids, raw = _fill(m, [(kb, vb)] * NL, D, H, lens, seed=31)
    B = len(lens)
    q, k_new, v_new = _step_inputs(NL, B, H, G, D, 3900)
    cache.extend(ids, [1] * B)
    out = cache.decode_layers(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    for l in range(NL):
        for s in ids:
            _check_row(cache, l, s, lens[s], k_new[l, s:s + 1], v_new[l, s:s + 1], kb, vb)
        ref = _reference(q[l], raw, l, ids, kb, vb, k_new[l], v_new[l])
        assert_close_attention(out[l], ref, f"layer {l}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (16, 16)])
def test_layer_batched_step_over_a_rotating_window(kb, vb):
    """A windowed sequence (its ring wrapped) beside an unwindowed one, two layers in one call."""
    m = kvq()
    D, H, G, P, W, NL = 64, 2, 8, 64, 256, 2
    cache = m.Cache(n_layers=NL, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=2,
                    max_tokens=64 * 40, page_tokens=P, max_seq_tokens=64 * 24)
    cache.set_window(0, W)
    ids = [0, 1]
    hist = {(l, s): ([], []) for l in range(NL) for s in ids}
    for step, chunk in enumerate([250, 200, 150, 100]):   # an append never exceeds the window
        n = [chunk, chunk // 3]
        cache.extend(ids, n)
        for l in range(NL):
            ks = [decode_kv(x, H, D, 100 * step + 10 * l + s) for s, x in enumerate(n)]
            vs = [random_fp16((x, H, D), 5000 + 100 * step + 10 * l + s) for s, x in enumerate(n)]
            cache.append(l, ids, n, torch.cat(ks).cuda(), torch.cat(vs).cuda())
            for s in ids:
                hist[(l, s)][0].append(ks[s])
                hist[(l, s)][1].append(vs[s])
    cache.extend(ids, [1, 1])
    q, k_new, v_new = _step_inputs(NL, 2, H, G, D, 4900)
    out = cache.decode_layers(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    for l in range(NL):
        ref = []
        for s, w in zip(ids, (W, 0)):
            k = torch.cat(hist[(l, s)][0] + [k_new[l, s:s + 1]])
            v = torch.cat(hist[(l, s)][1] + [v_new[l, s:s + 1]])
            ref.append(oracle.attention_decode_window(q[l, s].numpy(), oracle_dequant(k, kb), oracle_dequant(v, vb), w))
        assert_close_attention(out[l], np.stack(ref), f"layer {l} over the window")
    cache.close()


@pytest.mark.gpu
def test_layer_batched_step_replays_in_a_cuda_graph():
    """The layer-batched call only validates and enqueues: captured once, every replay gives the eager
    result bit for bit (the replayed step re-appends the same token at the same position)."""
    m = kvq()
    D, H, G, NL = 64, 4, 8, 4
    lens = [500, 8000]
    cache, ids, _ = _fill(m, [(8, 4)] * NL, D, H, lens, seed=41)
    B = len(lens)
    q, k_new, v_new = (t.cuda() for t in _step_inputs(NL, B, H, G, D, 5900))
    cache.extend(ids, [1] * B)
    out = torch.empty_like(q)
    ws = torch.empty(cache.decode_layers_workspace_size(NL, B, H * G), dtype=torch.uint8, device="cuda")
    eager = cache.decode_layers(0, ids, q, k_new, v_new, out=torch.empty_like(q), workspace=ws).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        cache.decode_layers(0, ids, q, k_new, v_new, out=out, workspace=ws)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    cache.check()
    del g
    cache.close()


@pytest.mark.gpu
def test_layer_batched_step_on_a_tensor_core_cache():
    """A cache created with the tensor-core decode flag: the layer-batched call runs the CUDA-core
    kernels (the flag applies to the per-layer calls) and matches the oracle; the per-layer calls on
    the twin cache (tensor-core kernel) match it too."""
    m = kvq()
    D, H, G, NL = 128, 8, 4, 2
    lens = [300, 2000]
    B = len(lens)

    def build():
        cache = m.Cache(n_layers=NL, n_kv_heads=H, head_dim=D, k_bits=8, v_bits=4, max_seqs=B,
                        max_tokens=sum(lens) + 512 * B, decode_tc=True)
        raw = {}
        cache.extend(list(range(B)), lens)
        for l in range(NL):
            ks = [decode_kv(n, H, D, 61 + 100 * s + l) for s, n in enumerate(lens)]
            vs = [random_fp16((n, H, D), 68 + 100 * s + l) for s, n in enumerate(lens)]
            cache.append(l, list(range(B)), lens, torch.cat(ks).cuda(), torch.cat(vs).cuda())
            for s in range(B):
                raw[(l, s)] = (ks[s], vs[s])
        return cache, raw

    cache, raw = build()
    twin, _ = build()
    ids = list(range(B))
    q, k_new, v_new = _step_inputs(NL, B, H, G, D, 6900)
    cache.extend(ids, [1] * B)
    out = cache.decode_layers(0, ids, q.cuda(), k_new.cuda(), v_new.cuda())
    cache.check()
    twin.extend(ids, [1] * B)
    for l in range(NL):
        sep = twin.decode_append(l, ids, q[l].cuda(), k_new[l].cuda(), v_new[l].cuda())
        ref = _reference(q[l], raw, l, ids, 8, 4, k_new[l], v_new[l])
        assert_close_attention(out[l], ref, f"layer-batched, layer {l}")
        assert_close_attention(sep, ref, f"per-layer tensor-core call, layer {l}")
        for s in ids:
            _check_row(cache, l, s, lens[s], k_new[l, s:s + 1], v_new[l, s:s + 1], 8, 4)
    twin.check()
    cache.close()
    twin.close()
