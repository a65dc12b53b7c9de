"""The seeded input recipe (shared by the oracle's tests and the CUDA path's
tests and benchmark): slices regenerate on their own, the outlier channels and
length draws follow the stated workload shapes."""
import torch

from asymmetric_quantized_kv_kvq_b200.inputs import (GEN_CHUNK, OUTLIER_SCALE, WORKLOADS, cached_lengths, gen_kv,
                                                     gen_q, outlier_channels, parse_precision, random_fp16, seed_for)


def test_a_slice_regenerates_on_its_own_across_chunk_boundaries():
    wl = WORKLOADS["tinyllama-22l-8k"]
    k_all, v_all = gen_kv(wl, 3, 0, 0, GEN_CHUNK + 300)
    k, v = gen_kv(wl, 3, 0, GEN_CHUNK - 100, 300)
    assert torch.equal(k, k_all[GEN_CHUNK - 100: GEN_CHUNK + 200])
    assert torch.equal(v, v_all[GEN_CHUNK - 100: GEN_CHUNK + 200])
    assert k.dtype == torch.float16 and k.shape == (300, wl.n_kv_heads, wl.head_dim)
    k0, _ = gen_kv(wl, 3, 0, 0, 0)
    assert k0.shape == (0, wl.n_kv_heads, wl.head_dim)


def test_layers_sequences_and_tensors_draw_different_values():
    wl = WORKLOADS["llama3-8b-b32-32k"]
    a, b = gen_kv(wl, 0, 0, 0, 64)
    c, _ = gen_kv(wl, 1, 0, 0, 64)
    d, _ = gen_kv(wl, 0, 1, 0, 64)
    assert not torch.equal(a, b) and not torch.equal(a, c) and not torch.equal(a, d)
    assert not torch.equal(gen_q(wl, 0, 0), gen_q(wl, 0, 1))
    assert seed_for(1, 2) == seed_for(1, 2) != seed_for(2, 1)


def test_outlier_channels_follow_the_workload_rule():
    tl = WORKLOADS["tinyllama-22l-8k"]
    m = outlier_channels(tl, 5)
    assert m.shape == (4, 64) and (m.sum(dim=1) == 4).all()          # 4 per (layer, KV head)
    ll = WORKLOADS["llama3-8b-b32-32k"]
    m = outlier_channels(ll, 7)
    assert m.shape == (8, 128) and int(m.sum()) == round(0.01 * 8 * 128)   # 1% of Hkv * D per layer
    assert not torch.equal(outlier_channels(ll, 7), outlier_channels(ll, 8))
    k, v = gen_kv(ll, 7, 0, 0, 4096)
    ks = k.float().std(dim=0)
    assert (ks[m] > 0.8 * OUTLIER_SCALE).all() and (ks[~m] < 1.2).all()    # keys x10 on those channels only
    assert (v.float().std(dim=0) < 1.2).all()                              # values have no outliers


def test_prefill_lengths_and_precisions():
    wl = WORKLOADS["prefill-16x4096"]
    lens = cached_lengths(wl)
    assert lens == cached_lengths(wl) and len(lens) == 16
    assert all(wl.cached_lo <= t <= wl.cached_hi for t in lens) and len(set(lens)) > 8
    assert cached_lengths(WORKLOADS["llama3-8b-b32-32k"]) == [32768] * 32
    assert parse_precision("K8V4") == (8, 4) and parse_precision("fp16") == (16, 16)
    assert parse_precision("K4V8") == (4, 8)
    assert torch.equal(random_fp16((3, 5), 9), random_fp16((3, 5), 9))
