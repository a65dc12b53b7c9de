"""GPU parity of per-layer precision (the KVSplit page's roadmap item "Layer-Specific
Quantization"): one cache whose layers are K8V4, K4V8, FP16, K8V8 and K4V4.  Every layer's
appended codes and scales are bit-exact against the oracle's quantiser at that layer's bit
widths, and decode, the fused one-token step and chunked prefill of every layer match the
oracle's float64 attention over that layer's dequantisation."""

import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, oracle_export, assert_close_attention

LAYERS = [(8, 4), (4, 8), (16, 16), (8, 8), (4, 4)]


@pytest.mark.gpu
@pytest.mark.parametrize("D,H,G", [(128, 2, 4), (64, 4, 8)])
def test_mixed_layer_precision_matches_oracle(D, H, G):
    m = kvq()
    lens = [300, 37, 1000]
    B, L = len(lens), len(LAYERS)
    cache = m.Cache(n_layers=L, n_kv_heads=H, head_dim=D, k_bits=8, v_bits=4, max_seqs=B,
                    max_tokens=sum(lens) + 512 * B, layer_bits=LAYERS)
    ids = list(range(B))
    cache.extend(ids, lens)
    raw = {}
    for layer in range(L):
        ks = [decode_kv(n, H, D, 1000 * layer + s) for s, n in enumerate(lens)]
        vs = [random_fp16((n, H, D), 1000 * layer + 50 + s) for s, n in enumerate(lens)]
        cache.append(layer, ids, lens, torch.cat(ks).cuda(), torch.cat(vs).cuda())
        for s in ids:
            raw[(layer, s)] = [ks[s], vs[s]]
    # footprint: the per-layer closed form
    assert cache.footprint()[1] == sum(oracle.footprint_bytes_layers(H, D, LAYERS, n) for n in lens)
    for layer, (kb, vb) in enumerate(LAYERS):
        # stored rows, bit for bit
        for s in ids:
            exp = cache.export(layer, s, 0, lens[s])
            for name, x, bits in (("k", raw[(layer, s)][0], kb), ("v", raw[(layer, s)][1], vb)):
                codes, scales = oracle_export(x, bits)
                got = exp[f"{name}_codes"].cpu().numpy()
                if bits == 16:
                    assert (got.view(np.uint16) == codes.view(np.uint16)).all(), f"layer {layer} {name}"
                else:
                    assert (got == codes).all(), f"layer {layer} {name} codes"
                    assert (exp[f"{name}_scales"].cpu().numpy().view(np.uint16) == scales.view(np.uint16)).all()
        # decode
        q = random_fp16((B, H * G, D), 7 + layer)
        out = cache.decode(layer, ids, q.cuda())
        ref = oracle.attention_decode_batch(
            q.numpy(), [(oracle_dequant(raw[(layer, s)][0], kb), oracle_dequant(raw[(layer, s)][1], vb)) for s in ids])
        assert_close_attention(out, ref, f"decode layer {layer} K{kb}V{vb}")
    cache.check()
    # one fused decode step per layer
    cache.extend(ids, [1] * B)
    for layer, (kb, vb) in enumerate(LAYERS):
        k1 = decode_kv(B, H, D, 5000 + layer)
        v1 = random_fp16((B, H, D), 6000 + layer)
        q = random_fp16((B, H * G, D), 7000 + layer)
        out = cache.decode_append(layer, ids, q.cuda(), k1.cuda(), v1.cuda())
        for s in ids:
            raw[(layer, s)][0] = torch.cat([raw[(layer, s)][0], k1[s:s + 1]])
            raw[(layer, s)][1] = torch.cat([raw[(layer, s)][1], v1[s:s + 1]])
        ref = oracle.attention_decode_batch(
            q.numpy(), [(oracle_dequant(raw[(layer, s)][0], kb), oracle_dequant(raw[(layer, s)][1], vb)) for s in ids])
        assert_close_attention(out, ref, f"decode step layer {layer} K{kb}V{vb}")
    cache.check()
    # a prefill chunk of 70 rows on every layer
    C = 70
    cache.extend(ids, [C] * B)
    for layer, (kb, vb) in enumerate(LAYERS):
        kc = [decode_kv(C, H, D, 8000 + 10 * layer + s) for s in ids]
        vc = [random_fp16((C, H, D), 9000 + 10 * layer + s) for s in ids]
        cache.append(layer, ids, [C] * B, torch.cat(kc).cuda(), torch.cat(vc).cuda())
        q = random_fp16((B * C, H * G, D), 9500 + layer)
        out = cache.prefill(layer, ids, [C] * B, q.cuda())
        for s in ids:
            k = torch.cat([raw[(layer, s)][0], kc[s]])
            v = torch.cat([raw[(layer, s)][1], vc[s]])
            n_cached = k.shape[0] - C
            ref = oracle.attention_prefill(q[s * C:(s + 1) * C].numpy(), oracle_dequant(k, kb), oracle_dequant(v, vb),
                                           n_cached)
            assert_close_attention(out[s * C:(s + 1) * C], ref, f"prefill layer {layer} K{kb}V{vb} seq {s}")
    cache.check()
    cache.close()
