"""The code rounding of the append and fused-append kernels (quant_block.cuh: round_mag), restated in
float64 NumPy and checked against roundf of the IEEE fp32 quotient: n = rint_even(fp32 FMA(|x|,
fp32(1 / |d|), 1.5 2^23) - 1.5 2^23), one upward step when the exact remainder |x| - n |d| reaches
|d| / 2, and the remainder never below -|d| / 2.  Every fp16 magnitude with |x| / |d| <= 128.5 (both
code widths' range) against every 8th positive finite fp16 scale; KVQ_ROUND_ALL_SCALES=1 takes all of
them (7.0e8 pairs, under a minute)."""
import os

import numpy as np


def test_one_sided_correction_matches_ieee_roundf():
    h = np.arange(0x0000, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)   # finite fp16 >= 0
    ds = h[h > 0]
    if os.environ.get("KVQ_ROUND_ALL_SCALES") != "1":
        ds = ds[::8]
    M = 1.5 * 2.0**23
    checked = 0
    for i in range(0, len(ds), 64):
        d = ds[i:i + 64][:, None]
        ra = (1.0 / d.astype(np.float32)).astype(np.float32).astype(np.float64)        # fp32 reciprocal
        sel = h[None, :] <= 128.5 * d
        ax = np.broadcast_to(h[None, :], sel.shape)
        n = ((ax * ra + M).astype(np.float32).astype(np.float64)) - M                     # one fp32 rounding
        e = ax - n * d                                                                     # exact
        assert not np.any(sel & (e < -0.5 * d)), "remainder below -|d|/2"
        n1 = n + (e >= 0.5 * d)
        q = (ax.astype(np.float32) / np.broadcast_to(d, sel.shape).astype(np.float32)).astype(np.float64)
        ref = np.floor(q + 0.5)                                                            # roundf, q >= 0
        assert not np.any(sel & (n1 != ref)), "rounded code differs from roundf of the IEEE quotient"
        checked += int(np.count_nonzero(sel))
    assert checked > 8e7
