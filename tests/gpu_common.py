"""Shared helpers of the GPU parity tests (not collected by pytest)."""
import numpy as np
import torch

import oracle
from asymmetric_quantized_kv_kvq_b200 import build as kbuild
from asymmetric_quantized_kv_kvq_b200.inputs import random_fp16

ATOL, RTOL = 2e-3, 1e-2      # attention: |gpu - ref| <= ATOL + RTOL * |ref| elementwise


def kvq():
    kbuild.build()
    from asymmetric_quantized_kv_kvq_b200 import kvq as m
    m.load_library()
    return m


def edge_kv(n: int, H: int, D: int, seed: int) -> torch.Tensor:
    """fp16 [n, H, D] ~ N(0, 1) with outlier channels x10 and, when there is
    room, special blocks: zeros, +/- ties of the largest magnitude, exact
    half-integer quotients, subnormal-range scales and fp16 extremes."""
    x = random_fp16((n, H, D), seed).float()
    x[:, :, 3] *= 10
    x[:, :, D - 5] *= 10
    specials = []
    z = torch.zeros(32)
    specials.append(z.clone())                                  # zero block
    t = torch.zeros(32); t[3], t[10] = -4.0, 4.0; specials.append(t)   # 4-bit sign tie
    t = torch.zeros(32); t[7], t[20] = 4.0, -4.0; specials.append(t)
    t = torch.arange(32, dtype=torch.float32) - 15.5; t[0] = 127.0; specials.append(t)  # x/d = k + .5
    specials.append(random_fp16((32,), seed + 1).float() * 1e-5)  # subnormal-range scale
    t = torch.full((32,), 65504.0); t[1::2] = -65504.0; specials.append(t)
    specials.append(random_fp16((32,), seed + 2).float() * 3000.0)
    k = 0
    for tok in range(n):
        for h in range(H):
            if (tok * H + h) % 7 == 3 and k < 4 * len(specials):
                b = (tok + h) % (D // 32)
                x[tok, h, 32 * b: 32 * b + 32] = specials[k % len(specials)]
                k += 1
    return x.to(torch.float16)


def oracle_export(x: torch.Tensor, bits: int):
    """Canonical (codes, scales) of fp16 [T, H, D] from the oracle."""
    return oracle.quantize_kv(x.cpu().numpy(), bits)


def oracle_dequant(x: torch.Tensor, bits: int) -> np.ndarray:
    c, s = oracle.quantize_kv(x.cpu().numpy(), bits)
    return oracle.dequantize_kv(c, s, bits)


def assert_close_attention(got: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} elements out of tolerance; worst at {i}: "
                             f"gpu {g[i]!r} ref {ref[i]!r}; max abs err {err.max():.3e}")
    return float(err.max()), float((err / np.maximum(np.abs(ref), 1e-30)).max())


def decode_kv(n: int, H: int, D: int, seed: int) -> torch.Tensor:
    """fp16 [n, H, D] ~ N(0, 1) with two key outlier channels x10 and a few
    zero / sign-tie blocks (no extreme magnitudes, so no single token
    dominates every softmax)."""
    x = random_fp16((n, H, D), seed).float()
    x[:, :, 3] *= 10
    x[:, :, D - 5] *= 10
    for tok in range(0, n, 11):
        h = tok % H
        b = (tok // 11) % (D // 32)
        if tok % 2:
            x[tok, h, 32 * b: 32 * b + 32] = 0.0
        else:
            x[tok, h, 32 * b + 3], x[tok, h, 32 * b + 10] = -4.0, 4.0
    return x.to(torch.float16)
