"""The code rounding of the append and fused-append kernels (quant_block.cuh: round_mag), restated in
float64 NumPy and checked against roundf of the IEEE fp32 quotient: n = floor(rd32(|x| ra + 1/2)) with
ra = 1 / |d| rounded up to fp32 and the FMA rounded down to fp32 (the kernels take the floor by adding
1.5 2^23 with rounding down).  Every fp16 magnitude with |x| / |d| <= 128.5 (both code widths' range)
against every 8th positive finite fp16 scale; KVQ_ROUND_ALL_SCALES=1 takes all of them (7.0e8 pairs,
under a minute)."""
import os

import numpy as np


def _round_down_f32(v):
    f = v.astype(np.float32)
    above = f.astype(np.float64) > v
    return np.where(above, np.nextafter(f, np.float32(-np.inf)), f).astype(np.float64)


def test_directed_rounding_matches_ieee_roundf():
    h = np.arange(0x0000, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)   # finite fp16 >= 0
    ds = h[h > 0]
    if os.environ.get("KVQ_ROUND_ALL_SCALES") != "1":
        ds = ds[::8]
    checked = 0
    for i in range(0, len(ds), 64):
        d = ds[i:i + 64][:, None]
        # fp32 reciprocal rounded up: the nearest fp32 to 1 / d, one step up when it lies below (the
        # product ra d is exact in float64, so the comparison with 1 is exact)
        ra = (1.0 / d).astype(np.float32)
        ra = np.where(ra.astype(np.float64) * d < 1.0, np.nextafter(ra, np.float32(np.inf)), ra).astype(np.float64)
        assert np.all(ra * d >= 1.0) and np.all(_round_down_f32(ra * (1 - 2.0**-30)) * d < 1.0)
        sel = h[None, :] <= 128.5 * d
        ax = np.broadcast_to(h[None, :], sel.shape)
        s = ax * ra + 0.5                                 # exact where it matters (t >= 1/2: under 44 bits)
        n = np.floor(_round_down_f32(s))                  # FMA rounded down, then the floor
        q = (ax.astype(np.float32) / np.broadcast_to(d, sel.shape).astype(np.float32)).astype(np.float64)
        ref = np.floor(q + 0.5)                           # roundf, q >= 0
        assert not np.any(sel & (n != ref)), "rounded code differs from roundf of the IEEE quotient"
        checked += int(np.count_nonzero(sel))
    assert checked > 8e7


def test_directed_rounding_is_sensitive_to_the_tie_handling():
    """The identity needs both directed roundings: with round-to-nearest for the reciprocal and the FMA
    some exact ties (t = k + 1/2) come out at k, so the check above would catch such a change."""
    h = np.arange(0x0000, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    d = h[h > 0][::97][:, None]
    ra = (1.0 / d).astype(np.float32).astype(np.float64)                              # nearest
    ax = np.broadcast_to(h[None, :], (d.shape[0], h.size))
    sel = ax <= 128.5 * d
    n = np.floor((ax * ra + 0.5).astype(np.float32).astype(np.float64))
    q = (ax.astype(np.float32) / np.broadcast_to(d, ax.shape).astype(np.float32)).astype(np.float64)
    assert np.any(sel & (n != np.floor(q + 0.5)))


def test_normal_scales_need_no_clamp():
    """The append kernel skips the clamps that a normal fp16 scale cannot reach: with |d| >= 2^-14,
    every 8-bit block has amax / d < 127.5 (d = fp16(fp32(amax / 127))), so no code rounds past 127,
    and every 4-bit block has |m| / |d| < 8.5 (d = fp16(m / -8)), so no code rounds below -8.  Subnormal
    scales do need them (their amax / d reaches 190 and |m| / |d| 11)."""
    h = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16)       # positive finite fp16
    a = h.astype(np.float64)
    d8 = (h.astype(np.float32) / np.float32(127.0)).astype(np.float16).astype(np.float64)
    n8 = d8 >= 2.0**-14
    assert np.all(2 * a[n8] < 255 * d8[n8])                          # amax < 127.5 d, exactly
    assert np.any(2 * a[(d8 > 0) & ~n8] >= 255 * d8[(d8 > 0) & ~n8])
    d4 = (h.astype(np.float32) * np.float32(0.125)).astype(np.float16).astype(np.float64)
    n4 = d4 >= 2.0**-14
    assert np.all(2 * a[n4] < 17 * d4[n4])                           # |m| < 8.5 |d|, exactly
    assert np.any(2 * a[(d4 > 0) & ~n4] >= 17 * d4[(d4 > 0) & ~n4])
