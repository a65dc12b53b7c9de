"""GPU parity of the rotating window (the [Reuse] page's rotating 8192-token cache, "O Que Nao
Funcionou"): a windowed sequence keeps a ring of pages and its query attends to the last W
positions only.  After the ring has wrapped several times, decode (both the quantized and the
fp16 kernels, and the fused one-token step) matches the oracle's attention_decode_window over the
sequence's whole token history, next to an unwindowed sequence in the same batch."""
import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, assert_close_attention


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (16, 16), (4, 8)])
@pytest.mark.parametrize("D,H,G", [(128, 2, 4), (64, 2, 8)])
def test_windowed_decode_matches_oracle(kb, vb, D, H, G):
    m = kvq()
    P, windows = 64, [256, 0, 512]
    cache = m.Cache(n_layers=1, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=3,
                    max_tokens=64 * 60, page_tokens=P, max_seq_tokens=64 * 24)
    for s, w in enumerate(windows):
        if w:
            cache.set_window(s, w)
    ids = [0, 1, 2]
    hist = {s: ([], []) for s in ids}
    rng = np.random.default_rng(kb * 10 + D)
    step = 0
    for chunk in [100, 1, 200, 37, 250, 5, 128, 64, 3, 190, 1, 1]:
        n = [chunk, min(chunk, 40), chunk]
        cache.extend(ids, n)
        ks = [decode_kv(x, H, D, 1000 + 10 * step + s) for s, x in enumerate(n)]
        vs = [random_fp16((x, H, D), 5000 + 10 * step + s) for s, x in enumerate(n)]
        cache.append(0, ids, n, torch.cat(ks).cuda(), torch.cat(vs).cuda())
        for s in ids:
            hist[s][0].append(ks[s])
            hist[s][1].append(vs[s])
        q = random_fp16((3, H * G, D), 9000 + step)
        out = cache.decode(0, ids, q.cuda())
        cache.check()
        ref = np.stack([oracle.attention_decode_window(
            q[s].numpy(), oracle_dequant(torch.cat(hist[s][0]), kb), oracle_dequant(torch.cat(hist[s][1]), vb),
            windows[s]) for s in ids])
        assert_close_attention(out, ref, f"step {step} lens {[cache.length(s) for s in ids]}")
        step += int(rng.integers(1, 3))
    assert cache.length(0) > 3 * 256                              # the ring wrapped several times
    # one fused step: append + decode in one launch over the window
    cache.extend(ids, [1, 1, 1])
    k1 = decode_kv(3, H, D, 77)
    v1 = random_fp16((3, H, D), 78)
    q = random_fp16((3, H * G, D), 79)
    out = cache.decode_append(0, ids, q.cuda(), k1.cuda(), v1.cuda())
    cache.check()
    for s in ids:
        hist[s][0].append(k1[s:s + 1])
        hist[s][1].append(v1[s:s + 1])
    ref = np.stack([oracle.attention_decode_window(
        q[s].numpy(), oracle_dequant(torch.cat(hist[s][0]), kb), oracle_dequant(torch.cat(hist[s][1]), vb),
        windows[s]) for s in ids])
    assert_close_attention(out, ref, "fused step over the window")
    # the stored window is bit-exact: export of the last 256 positions of sequence 0
    n0 = cache.length(0)
    exp = cache.export(0, 0, n0 - 256, 256)
    kc, _ = oracle.quantize_kv(torch.cat(hist[0][0])[-256:].numpy(), kb) if kb != 16 else (None, None)
    if kb != 16:
        assert (exp["k_codes"].cpu().numpy() == kc).all()
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", [(8, 4), (4, 8)])
def test_windowed_decode_256_token_stages(kb, vb):
    """The pages' 8192-token window on 256-token pages, in a step large enough for 256-token stages:
    two windowed sequences whose rings have wrapped (the window starts inside a chunk, so its first
    stage is masked) next to an unwindowed one, decode and the fused step against the oracle."""
    m = kvq()
    D, H, G, P, W = 128, 8, 4, 256, 8192
    cache = m.Cache(n_layers=1, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=3,
                    max_tokens=P * 140, page_tokens=P, max_seq_tokens=P * 48)
    cache.set_window(0, W)
    cache.set_window(2, W)
    ids = [0, 1, 2]
    hist = {s: ([], []) for s in ids}
    for step, n in enumerate([[4000, 4000, 3000], [4000, 4000, 3000], [3100, 2100, 2950]]):
        cache.extend(ids, n)
        ks = [decode_kv(x, H, D, 300 + 10 * step + s) for s, x in enumerate(n)]
        vs = [random_fp16((x, H, D), 700 + 10 * step + s) for s, x in enumerate(n)]
        cache.append(0, ids, n, torch.cat(ks).cuda(), torch.cat(vs).cuda())
        for s in ids:
            hist[s][0].append(ks[s])
            hist[s][1].append(vs[s])
    windows = [W, 0, W]
    q = random_fp16((3, H * G, D), 901)
    out = cache.decode(0, ids, q.cuda())
    cache.check()
    ref = np.stack([oracle.attention_decode_window(
        q[s].numpy(), oracle_dequant(torch.cat(hist[s][0]), kb), oracle_dequant(torch.cat(hist[s][1]), vb),
        windows[s]) for s in ids])
    assert_close_attention(out, ref, "256-token stages, windows")
    cache.extend(ids, [1, 1, 1])
    k1 = decode_kv(3, H, D, 911)
    v1 = random_fp16((3, H, D), 912)
    q = random_fp16((3, H * G, D), 913)
    out = cache.decode_append(0, ids, q.cuda(), k1.cuda(), v1.cuda())
    cache.check()
    for s in ids:
        hist[s][0].append(k1[s:s + 1])
        hist[s][1].append(v1[s:s + 1])
    ref = np.stack([oracle.attention_decode_window(
        q[s].numpy(), oracle_dequant(torch.cat(hist[s][0]), kb), oracle_dequant(torch.cat(hist[s][1]), vb),
        windows[s]) for s in ids])
    assert_close_attention(out, ref, "256-token stages, windows, fused step")
    cache.close()
