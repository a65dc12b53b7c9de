"""GPU parity: quantise-on-append must reproduce the oracle's codes and fp16
scales bit for bit (read back through the canonical export)."""
import numpy as np
import pytest
import torch

from gpu_common import kvq, edge_kv, oracle_export

FORMATS = [(8, 4), (8, 8), (4, 4), (4, 8), (16, 16)]


def _compare(cache, layer, seq, x_k, x_v, kb, vb):
    T = x_k.shape[0]
    got = cache.export(layer, seq, 0, T)
    torch.cuda.synchronize()
    for name, x, bits in (("k", x_k, kb), ("v", x_v, vb)):
        codes, scales = oracle_export(x, bits)
        gc = got[f"{name}_codes"].cpu().numpy()
        if bits == 16:
            assert (gc.view(np.uint16) == codes.view(np.uint16)).all(), f"{name} fp16 copy differs"
            continue
        assert gc.dtype == codes.dtype
        mism = np.argwhere(gc != codes)
        assert mism.size == 0, f"{name} codes differ at {mism[:5].tolist()} (of {len(mism)})"
        gs = got[f"{name}_scales"].cpu().numpy().view(np.uint16)
        mism = np.argwhere(gs != scales.view(np.uint16))
        assert mism.size == 0, f"{name} scales differ at {mism[:5].tolist()}"


@pytest.mark.gpu
@pytest.mark.parametrize("kb,vb", FORMATS)
@pytest.mark.parametrize("D,H", [(64, 3), (128, 2)])
def test_append_is_bit_exact(kb, vb, D, H):
    m = kvq()
    lens = [1, 31, 33, 255, 256, 257, 600]
    seqs = list(range(len(lens)))
    cache = m.Cache(n_layers=2, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=8,
                    max_tokens=16 * 1024)
    dev = torch.device("cuda")
    xs = {}
    # three rounds per sequence: a ragged chunk, one decode-like token, another chunk
    rounds = [[(L + 1) // 2 for L in lens], [1] * len(lens), [L - (L + 1) // 2 for L in lens]]
    for r, n_new in enumerate(rounds):
        ids = [s for s, n in zip(seqs, n_new) if n > 0]
        nn = [n for n in n_new if n > 0]
        cache.extend(ids, nn)
        for layer in range(2):
            ks = [edge_kv(n, H, D, 1000 * r + 10 * s + layer) for s, n in zip(ids, nn)]
            vs = [edge_kv(n, H, D, 5000 + 1000 * r + 10 * s + layer) for s, n in zip(ids, nn)]
            cache.append(layer, ids, nn, torch.cat(ks).to(dev), torch.cat(vs).to(dev))
            for s, kx, vx in zip(ids, ks, vs):
                pk, pv = xs.get((layer, s), (None, None))
                xs[(layer, s)] = (kx if pk is None else torch.cat([pk, kx]),
                                  vx if pv is None else torch.cat([pv, vx]))
    cache.check()
    for (layer, s), (kx, vx) in xs.items():
        assert kx.shape[0] == cache.length(s)
        _compare(cache, layer, s, kx, vx, kb, vb)
    cache.close()


@pytest.mark.gpu
def test_append_of_zero_new_tokens_is_a_noop():
    m = kvq()
    cache = m.Cache(1, 2, 64, 8, 4, max_seqs=2, max_tokens=512)
    cache.extend([0], [3])
    x = edge_kv(3, 2, 64, 7).cuda()
    cache.append(0, [0], [3], x, x)
    cache.append(0, [0], [0], None, None)
    cache.check()
    _compare(cache, 0, 0, x.cpu(), x.cpu(), 8, 4)
    cache.close()
