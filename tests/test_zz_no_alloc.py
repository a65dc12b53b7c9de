"""kvq_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory -- a plugin running inside an application that owns all GPU
memory and hands it only inputs and outputs, an engine whose allocator has
reserved the whole device, or a serving loop that must never call cudaMalloc /
cudaFree because they can synchronise the GPU.  Its split-KV scratch lives in
a fixed array inside the library, so its result must equal that of
kvq_decode_attn with a caller-owned workspace bit for bit (same kernel, same
plan, only the scratch address differs), call after call, whatever the array
held before.

This file is collected last on purpose: when it fails, a run that stops at the
first failure has already run every other test."""
import pytest
import torch

from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv


def _cache(m, lens, H=8, D=128, kb=8, vb=4):
    cache = m.Cache(n_layers=2, n_kv_heads=H, head_dim=D, k_bits=kb, v_bits=vb, max_seqs=len(lens),
                    max_tokens=sum(lens) + 256 * len(lens))
    ids = list(range(len(lens)))
    cache.extend(ids, lens)
    for layer in range(2):
        ks = torch.cat([decode_kv(L, H, D, 40 + 10 * s + layer) for s, L in enumerate(lens)])
        vs = torch.cat([random_fp16((L, H, D), 80 + 10 * s + layer) for s, L in enumerate(lens)])
        cache.append(layer, ids, lens, ks.cuda(), vs.cuda())
    return cache, ids


@pytest.mark.gpu
def test_noalloc_decode_matches_the_workspace_entry_point_on_consecutive_calls():
    m = kvq()
    lens = [700, 3000, 45, 1, 20011]           # short items and items split over many CTAs
    cache, ids = _cache(m, lens)
    H, G, D = 8, 4, 128
    q0 = random_fp16((len(lens), H * G, D), 3).cuda()
    q1 = random_fp16((len(lens), H * G, D), 4).cuda()
    ref0 = cache.decode(0, ids, q0)
    ref1 = cache.decode(1, ids, q1)
    torch.cuda.synchronize()
    # two calls in a row with the same inputs, then one with other inputs
    for _ in range(2):
        got = cache.decode_noalloc(0, ids, q0)
        torch.cuda.synchronize()
        assert torch.equal(got, ref0)
    got = cache.decode_noalloc(1, ids, q1)
    torch.cuda.synchronize()
    assert torch.equal(got, ref1)
    cache.check()
    cache.close()


def test_noalloc_rejects_batches_beyond_the_fixed_scratch():
    m = kvq()
    # host-only cache: the size check happens before anything touches a GPU
    c = m.Cache(n_layers=1, n_kv_heads=8, head_dim=128, k_bits=8, v_bits=4, max_seqs=256, max_tokens=1 << 16,
                host_only=True)
    need = c.decode_workspace_size(256, 64)
    assert need > m.KVQ_NOALLOC_SCRATCH_BYTES
    ids = list(range(256))
    c.extend(ids, [1] * 256)
    lib = m.load_library()
    import ctypes
    arr = (ctypes.c_int32 * 256)(*ids)
    st = lib.kvq_decode_attn_noalloc(c._h, 0, 256, arr, 64, 16, 16, 0.0, None)
    assert st == 7                                                     # KVQ_ERR_WORKSPACE
    assert b"KVQ_NOALLOC_SCRATCH_BYTES" in lib.kvq_last_error()
    c.close()


def test_noalloc_refuses_a_host_only_cache_before_touching_a_device():
    """A host-only cache with a batch that fits is refused with KVQ_ERR_UNSUPPORTED before the
    scratch array's device address is looked up (no CUDA call is made)."""
    m = kvq()
    c = m.Cache(n_layers=1, n_kv_heads=8, head_dim=128, k_bits=8, v_bits=4, max_seqs=4, max_tokens=4096,
                host_only=True)
    c.extend([0], [10])
    lib = m.load_library()
    import ctypes
    arr = (ctypes.c_int32 * 1)(0)
    assert lib.kvq_decode_attn_noalloc(c._h, 0, 1, arr, 32, 16, 16, 0.0, None) == 2   # KVQ_ERR_UNSUPPORTED
    assert b"host-only" in lib.kvq_last_error()
    c.close()
