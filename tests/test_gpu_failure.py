"""Failure detection on the GPU without a GPU fault: a cache created with the test hook
KVQ_TEST_WITHHOLD_ARRIVAL=1 runs the quantized decode kernel with CTA 0's first stage never
filled and every bounded wait limited to 1 ms.  The waits run out, the kernel records
kErrWaitTimeout in the cache's device error word and returns (no trap, no fault, no hang);
kvq_cache_check reports KVQ_ERR_DEVICE_CHECK with that code, and the CUDA context stays usable:
the next decode on a normal cache matches the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16
from gpu_common import kvq, decode_kv, oracle_dequant, assert_close_attention

K_ERR_WAIT_TIMEOUT = 0x100


def _filled(m, lens, H, D):
    cache = m.Cache(n_layers=1, n_kv_heads=H, head_dim=D, k_bits=8, v_bits=4, max_seqs=len(lens),
                    max_tokens=sum(lens) + 256 * len(lens))
    ids = list(range(len(lens)))
    cache.extend(ids, lens)
    ks = [decode_kv(L, H, D, 10 + s) for s, L in enumerate(lens)]
    vs = [random_fp16((L, H, D), 20 + s) for s, L in enumerate(lens)]
    cache.append(0, ids, lens, torch.cat(ks).cuda(), torch.cat(vs).cuda())
    return cache, ids, ks, vs


@pytest.mark.gpu
def test_a_withheld_arrival_times_out_and_is_reported(monkeypatch):
    m = kvq()
    H, G, D = 8, 4, 128
    lens = [3000, 500]
    monkeypatch.setenv("KVQ_TEST_WITHHOLD_ARRIVAL", "1")
    bad, ids, _, _ = _filled(m, lens, H, D)
    monkeypatch.delenv("KVQ_TEST_WITHHOLD_ARRIVAL")
    q = random_fp16((len(lens), H * G, D), 5).cuda()
    bad.decode(0, ids, q)                                   # enqueued fine; the kernel gives up on the device
    lib = m.load_library()
    detail = ctypes.c_uint32()
    st = lib.kvq_cache_check(bad._h, torch.cuda.current_stream().cuda_stream, ctypes.byref(detail))
    assert st == 6, f"expected KVQ_ERR_DEVICE_CHECK, got {st}"   # KVQ_ERR_DEVICE_CHECK
    assert detail.value & 0xF00 == K_ERR_WAIT_TIMEOUT, hex(detail.value)
    assert lib.kvq_cache_check(bad._h, torch.cuda.current_stream().cuda_stream, ctypes.byref(detail)) == 0
    bad.close()
    # the context is intact: a normal cache decodes correctly right after
    good, ids, ks, vs = _filled(m, lens, H, D)
    out = good.decode(0, ids, q)
    good.check()
    ref = oracle.attention_decode_batch(q.cpu().numpy(), [(oracle_dequant(k, 8), oracle_dequant(v, 4))
                                                          for k, v in zip(ks, vs)])
    assert_close_attention(out, ref, "after a reported timeout")
    good.close()
