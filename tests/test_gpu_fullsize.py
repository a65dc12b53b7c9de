"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (same batch, lengths, heads and kernel instantiation; one
layer, since every layer is an identical, independent launch).  The oracle
checks sampled outputs one by one: codes and scales of sampled sequences bit
for bit, attention of sampled sequences / rows within the suite tolerance.
Inputs come from the seeded generator on the GPU; the sampled slices are
copied to the host for the oracle."""
import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import (WORKLOADS, GEN_CHUNK, gen_kv, gen_q, gen_q_chunk,
                                                      cached_lengths, parse_precision)
from gpu_common import kvq, assert_close_attention


def _fill(cache, wl, ids, lens, keep):
    """Append every sequence's K / V chunk by chunk (layer 0); return host copies of `keep`."""
    host = {b: ([], []) for b in keep}
    for c in range(-(-max(lens) // GEN_CHUNK)):
        sel = [b for b in ids if lens[b] > c * GEN_CHUNK]
        n = [min(GEN_CHUNK, lens[b] - c * GEN_CHUNK) for b in sel]
        cache.extend(sel, n)
        kv = [gen_kv(wl, 0, b, c * GEN_CHUNK, m, device="cuda") for b, m in zip(sel, n)]
        cache.append(0, sel, n, torch.cat([k for k, _ in kv]), torch.cat([v for _, v in kv]))
        for b, (k, v) in zip(sel, kv):
            if b in host:
                host[b][0].append(k.cpu())
                host[b][1].append(v.cpu())
    return {b: (torch.cat(h[0]), torch.cat(h[1])) for b, h in host.items()}


def _check_codes(cache, b, k, v, kb, vb, tok0=0):
    T = k.shape[0]
    got = cache.export(0, b, tok0, T)
    torch.cuda.synchronize()
    for name, x, bits in (("k", k, kb), ("v", v, vb)):
        codes, scales = oracle.quantize_kv(x.numpy(), bits)
        gc = got[f"{name}_codes"].cpu().numpy()
        if bits == 16:
            assert (gc.view(np.uint16) == codes.view(np.uint16)).all()
        else:
            assert (gc == codes).all(), f"{name} codes differ for sequence {b}"
            assert (got[f"{name}_scales"].cpu().numpy().view(np.uint16) == scales.view(np.uint16)).all()


def _decode_case(name, precision, sample):
    m = kvq()
    wl = WORKLOADS[name]
    kb, vb = parse_precision(precision)
    B, T = wl.batch, wl.cached + 1            # the bench's first timed step sees T + 1 tokens
    cache = m.Cache(1, wl.n_kv_heads, wl.head_dim, kb, vb, max_seqs=B, max_tokens=B * (-(-T // 256)) * 256)
    ids = list(range(B))
    host = _fill(cache, wl, ids, [T] * B, sample)
    q = gen_q(wl, 0, 0, device="cuda")
    out = cache.decode(0, ids, q)
    cache.check()
    for b in sample:
        k, v = host[b]
        _check_codes(cache, b, k[-300:], v[-300:], kb, vb, tok0=T - 300)
        kh = oracle.dequantize_kv(*oracle.quantize_kv(k.numpy(), kb), kb)
        vh = oracle.dequantize_kv(*oracle.quantize_kv(v.numpy(), vb), vb)
        ref = oracle.attention_decode(q[b].cpu().numpy(), kh, vh)
        assert_close_attention(out[b], ref, f"{name} {precision} sequence {b}")
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("precision", ["FP16", "K8V8", "K8V4", "K4V4"])
def test_fullsize_tinyllama_22l_8k(precision):
    _decode_case("tinyllama-22l-8k", precision, [0])


@pytest.mark.gpu
def test_fullsize_llama3_batched_decode():
    _decode_case("llama3-8b-b32-32k", "K8V4", [0, 13, 31])


@pytest.mark.gpu
@pytest.mark.parametrize("precision", ["K8V4", "FP16"])
def test_fullsize_long_context_decode(precision):
    _decode_case("llama70b-b1-128k", precision, [0])


@pytest.mark.gpu
def test_fullsize_ragged_prefill():
    m = kvq()
    wl = WORKLOADS["prefill-16x4096"]
    kb, vb = parse_precision("K8V4")
    T = cached_lengths(wl)
    C = wl.chunk
    n = len(T)
    ids = list(range(n))
    sample = [int(np.argmax(T)), int(np.argmin(T)), 5]
    cache = m.Cache(1, wl.n_kv_heads, wl.head_dim, kb, vb, max_seqs=n,
                    max_tokens=sum(-(-(t + C) // 256) * 256 for t in T), max_seq_tokens=max(T) + C)
    host = _fill(cache, wl, ids, [t + C for t in T], sample)
    # rewind to the cached prefixes, then append the chunk as the benchmark does
    for b in ids:
        cache.truncate(b, T[b])
    cache.extend(ids, [C] * n)
    kv = [gen_kv(wl, 0, b, T[b], C, device="cuda") for b in ids]
    cache.append(0, ids, [C] * n, torch.cat([k for k, _ in kv]), torch.cat([v for _, v in kv]))
    q = torch.cat([gen_q_chunk(wl, 0, b, C, device="cuda") for b in ids])
    out = cache.prefill(0, ids, [C] * n, q)
    cache.check()
    rows = [0, 1, 31, 32, 2047, 4064, 4095]
    for b in sample:
        k, v = host[b]
        _check_codes(cache, b, k[T[b]:], v[T[b]:], kb, vb, tok0=T[b])
        kh = oracle.dequantize_kv(*oracle.quantize_kv(k.numpy(), kb), kb)
        vh = oracle.dequantize_kv(*oracle.quantize_kv(v.numpy(), vb), vb)
        qb = q[b * C:(b + 1) * C].cpu().numpy()
        ref = oracle.attention_prefill(qb, kh, vh, T[b], rows=rows)
        got = out[b * C:(b + 1) * C][rows]
        assert_close_attention(got, ref, f"prefill sequence {b} (cached {T[b]})")
    cache.close()
