"""Float64 CPU oracle: block quantisation, KV footprint and softmax attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).  No CUDA, no shared code
with the GPU path.

Pages (cited by title and section):
  [KVSplit]  "KVSplit - contexto 2 a 3 vezes mais longo em Apple Silicon",
             pt.news.hada.io/topic?id=20969
  [Reuse]    "Reutilizacao de Cache KV para Conversas Longas no Apple Silicon",
             openclawradar.com

Storage format (a reading of [KVSplit], "Uso de memoria conforme o comprimento
da sequencia": the printed MB column is exact for 32-element blocks that carry
one fp16 scale each, 34 B per 8-bit block and 18 B per 4-bit block; 18 B leaves
no room for a zero point, so blocks are symmetric, scale-only):

  Q8 block  amax = max|x_j|; d = fp16_rne(fp32_rn(amax / 127));
            c_j = clamp(round_half_away(fp32_rn(x_j / d)), -127, 127); d == 0 -> c = 0.
            x^_j = d * c_j.
  Q4 block  m = the x_j of largest |x_j| (lowest index on ties);
            d = fp16_rne(m / -8);
            c_j = clamp(round_half_away(fp32_rn(x_j / d)), -8, 7); d == 0 -> c = 0;
            stored nibble u_j = c_j + 8; byte i (0..15) = u_i | u_{i+16} << 4.
            x^_j = d * (u_j - 8).
  FP16      stored as is.

Attention ([KVSplit], "Exemplos de uso e opcoes de CLI": the cache is read
through the flash-attention path; flash attention computes exact softmax
attention):  query head h reads KV head h // (Hq / Hkv);
  s_t = sigma * sum_j q_j k^_{t,j},  sigma = 1/sqrt(D) unless given,
  p_t = exp(s_t - max s) / sum exp(.),  o = sum_t p_t v^_t,
over the dequantised cache.  Decode: the query at position T-1 sees tokens
0..T-1.  Chunked prefill ([Reuse], "Principais Descobertas e Benchmarks": keep
the cache and process only the new tokens): chunk row i, at absolute position
n_cached + i, sees tokens 0..n_cached+i, the chunk's own (already quantised)
tokens included.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "QK", "MIB", "block_bytes", "kv_bytes_per_token_layer", "footprint_bytes", "footprint_bytes_layers",
    "used_bytes",
    "q8_scale", "q4_scale", "round_half_away", "quantize_q8", "quantize_q4",
    "dequantize_q8", "dequantize_q4", "unpack_q4", "quantize_kv", "dequantize_kv",
    "attention_decode", "attention_decode_window", "attention_prefill", "attention_decode_batch", "lse_merge",
]

QK = 32            # elements per quantisation block
MIB = 1 << 20


# ---------------------------------------------------------------------------
# Footprint  ([KVSplit] "Uso de memoria conforme o comprimento da sequencia";
# pinned by the printed MB table at 8192 / 4096 / 128 tokens)
# ---------------------------------------------------------------------------
def block_bytes(bits: int, n_elements: int) -> int:
    """Stored bytes for n_elements values at `bits` (n a multiple of 32 for 4/8)."""
    if bits == 16:
        return 2 * n_elements
    if n_elements % QK:
        raise ValueError("quantised rows are whole 32-element blocks")
    if bits == 8:
        return (n_elements // QK) * (QK + 2)        # 32 int8 codes + fp16 scale = 34 B
    if bits == 4:
        return (n_elements // QK) * (QK // 2 + 2)   # 16 B of nibbles + fp16 scale = 18 B
    raise ValueError(f"unsupported bit width {bits}")


def kv_bytes_per_token_layer(n_kv_heads: int, head_dim: int, k_bits: int, v_bits: int) -> int:
    """K plus V bytes one token occupies in one layer."""
    n = n_kv_heads * head_dim
    return block_bytes(k_bits, n) + block_bytes(v_bits, n)


def used_bytes(n_layers, n_kv_heads, head_dim, k_bits, v_bits, n_tokens) -> int:
    """Bytes of the tokens actually held (no page rounding)."""
    return n_layers * n_tokens * kv_bytes_per_token_layer(n_kv_heads, head_dim, k_bits, v_bits)


def footprint_bytes(n_layers, n_kv_heads, head_dim, k_bits, v_bits, n_tokens,
                    page_tokens: int = 256) -> int:
    """Allocated bytes: capacity is whole pages of `page_tokens` tokens.

    The pages' 128-token row (5.50 / 2.23 / 1.55 MB) equals the closed form at a
    256-token capacity, which is the reading that fixes page_tokens = 256
    ([KVSplit] "Otimizacao para Apple Silicon e limitacoes" also attributes the
    gap between real and theoretical savings to page alignment).
    """
    pages = -(-n_tokens // page_tokens)
    return used_bytes(n_layers, n_kv_heads, head_dim, k_bits, v_bits, pages * page_tokens)


def footprint_bytes_layers(n_kv_heads, head_dim, layer_bits, n_tokens, page_tokens: int = 256) -> int:
    """Allocated bytes of a cache whose layers have their own (k_bits, v_bits)
    ([KVSplit] "Configuracao recomendada e roadmap": layer-specific quantisation,
    different precisions per layer).  Every layer holds the same tokens in whole
    pages, so the footprint is the sum of the single-layer footprints.
    Pinned by the printed table: a 22-layer cache half K8V4, half K4V4 holds
    (71.50 + 49.50) / 2 MB at 8192 tokens."""
    return sum(footprint_bytes(1, n_kv_heads, head_dim, kb, vb, n_tokens, page_tokens) for kb, vb in layer_bits)


# ---------------------------------------------------------------------------
# Block quantisation
# ---------------------------------------------------------------------------
def _check_fp16_blocks(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype != np.float16:
        raise TypeError("blocks are fp16 values")
    if x.shape[-1] != QK:
        raise ValueError("last axis must be one 32-element block")
    return x


def round_half_away(q: np.ndarray) -> np.ndarray:
    """Round to nearest integer, ties away from zero (C roundf).  q is float64
    holding fp32 values, so q +/- 0.5 is exact."""
    q = np.asarray(q, dtype=np.float64)
    return np.where(q >= 0, np.floor(q + 0.5), -np.floor(-q + 0.5))


def q8_scale(amax_f16: np.ndarray) -> np.ndarray:
    """d = fp16_rne(fp32_rn(amax / 127)).  Pinned exhaustively against exact
    rational rounding over every non-negative finite fp16 amax."""
    a = np.asarray(amax_f16, dtype=np.float16).astype(np.float32)
    return (a / np.float32(127.0)).astype(np.float16)


def q4_scale(m_f16: np.ndarray) -> np.ndarray:
    """d = fp16_rne(m / -8) for the signed largest-magnitude element m."""
    m = np.asarray(m_f16, dtype=np.float16).astype(np.float32)
    return (m / np.float32(-8.0)).astype(np.float16)


def _codes(x: np.ndarray, d: np.ndarray, lo: int, hi: int) -> np.ndarray:
    xf = x.astype(np.float32)
    df = d.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (xf / df).astype(np.float64)           # correctly rounded fp32 quotient
        c = np.clip(round_half_away(q), lo, hi)
    c = np.where(df == 0, 0.0, c)
    return c.astype(np.int64)


def quantize_q8(x):
    """8-bit block: returns (int8 codes [..., 32], fp16 scales [...])."""
    x = _check_fp16_blocks(x)
    amax = np.max(np.abs(x), axis=-1)
    d = q8_scale(amax)
    return _codes(x, d, -127, 127).astype(np.int8), d


def quantize_q4(x):
    """4-bit block: returns (packed uint8 [..., 16], fp16 scales [...]).
    Byte i holds element i in its low nibble and element i+16 in its high nibble."""
    x = _check_fp16_blocks(x)
    idx = np.argmax(np.abs(x), axis=-1)             # first maximum = lowest index
    m = np.take_along_axis(x, idx[..., None], axis=-1)[..., 0]
    d = q4_scale(m)
    u = (_codes(x, d, -8, 7) + 8).astype(np.uint8)
    packed = (u[..., :16] | (u[..., 16:] << 4)).astype(np.uint8)
    return packed, d


def dequantize_q8(codes, d) -> np.ndarray:
    return np.asarray(codes).astype(np.float64) * np.asarray(d, np.float16).astype(np.float64)[..., None]


def unpack_q4(packed) -> np.ndarray:
    """Signed codes c_j = u_j - 8, [..., 32], from packed bytes [..., 16]."""
    p = np.asarray(packed, dtype=np.uint8)
    u = np.concatenate([p & 0x0F, p >> 4], axis=-1).astype(np.int64)
    return u - 8


def dequantize_q4(packed, d) -> np.ndarray:
    return unpack_q4(packed).astype(np.float64) * np.asarray(d, np.float16).astype(np.float64)[..., None]


def quantize_kv(x, bits: int):
    """Quantise a [T, H, D] fp16 K or V tensor in 32-element blocks along D.

    Returns the canonical stored form (codes, scales):
      bits 16: (fp16 [T, H, D], None)
      bits 8 : (int8 [T, H, D], fp16 [T, H, D/32])
      bits 4 : (uint8 [T, H, D/2] packed per block, fp16 [T, H, D/32])
    """
    x = np.asarray(x)
    if x.dtype != np.float16 or x.ndim != 3:
        raise ValueError("expected fp16 [T, H, D]")
    T, H, D = x.shape
    if bits == 16:
        return x.copy(), None
    if D % QK:
        raise ValueError("head_dim must be a multiple of 32")
    blocks = x.reshape(T, H, D // QK, QK)
    if bits == 8:
        c, d = quantize_q8(blocks)
        return c.reshape(T, H, D), d
    if bits == 4:
        p, d = quantize_q4(blocks)
        return p.reshape(T, H, D // 2), d
    raise ValueError(f"unsupported bit width {bits}")


def dequantize_kv(codes, scales, bits: int) -> np.ndarray:
    """Canonical stored form -> float64 [T, H, D]."""
    codes = np.asarray(codes)
    if bits == 16:
        return codes.astype(np.float64)
    T, H = codes.shape[:2]
    if bits == 8:
        D = codes.shape[2]
        return dequantize_q8(codes.reshape(T, H, D // QK, QK), scales).reshape(T, H, D)
    if bits == 4:
        D = codes.shape[2] * 2
        return dequantize_q4(codes.reshape(T, H, D // QK, QK // 2), scales).reshape(T, H, D)
    raise ValueError(f"unsupported bit width {bits}")


# ---------------------------------------------------------------------------
# Attention over the dequantised cache
# ---------------------------------------------------------------------------
def attention_decode(q, k_hat, v_hat, scale=None) -> np.ndarray:
    """One query position: q [Hq, D], k_hat / v_hat [T, Hkv, D] -> o [Hq, D] (float64).
    Query head h uses KV head h // (Hq / Hkv)."""
    q = np.asarray(q).astype(np.float64)
    k_hat = np.asarray(k_hat, dtype=np.float64)
    v_hat = np.asarray(v_hat, dtype=np.float64)
    Hq, D = q.shape
    T, Hkv, _ = k_hat.shape
    if T == 0:
        raise ValueError("attention over an empty cache is undefined")
    G = Hq // Hkv
    sigma = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out = np.empty((Hq, D), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        s = (k_hat[:, g, :] @ q[h]) * sigma
        p = np.exp(s - s.max())
        out[h] = (p @ v_hat[:, g, :]) / p.sum()
    return out


def attention_decode_window(q, k_hat, v_hat, window: int, scale=None) -> np.ndarray:
    """Decode over a rotating cache of `window` tokens ([Reuse] "O Que Nao Funcionou":
    rotating the KV cache at 8192 tokens keeps only the most recent tokens, which
    gave the best tokens/s but lost the earlier context): the query at position
    T-1 sees only tokens max(0, T - window) .. T-1.  window = 0 means no window.
    Pinned by: window >= T gives attention_decode; window 1 gives the last
    token's value; brute force over the kept tokens on tiny inputs."""
    k_hat = np.asarray(k_hat, dtype=np.float64)
    v_hat = np.asarray(v_hat, dtype=np.float64)
    T = k_hat.shape[0]
    if window < 0:
        raise ValueError("window must be >= 0")
    lo = max(0, T - window) if window else 0
    return attention_decode(q, k_hat[lo:], v_hat[lo:], scale)


def attention_decode_batch(q, caches, scale=None) -> np.ndarray:
    """q [B, Hq, D]; caches = list of (k_hat, v_hat) per sequence."""
    return np.stack([attention_decode(q[b], k, v, scale) for b, (k, v) in enumerate(caches)])


def attention_prefill(q, k_hat, v_hat, n_cached: int, scale=None, rows=None) -> np.ndarray:
    """Causal chunk attention: q [C, Hq, D]; k_hat / v_hat [n_cached + C, Hkv, D].
    Row i (absolute position n_cached + i) sees tokens 0 .. n_cached + i.
    `rows` optionally restricts the computation to a subset of chunk rows
    (returned in that order)."""
    q = np.asarray(q)
    C = q.shape[0]
    if np.asarray(k_hat).shape[0] != n_cached + C:
        raise ValueError("cache must hold n_cached + C tokens")
    rows = range(C) if rows is None else rows
    return np.stack([attention_decode(q[i], k_hat[: n_cached + i + 1], v_hat[: n_cached + i + 1], scale)
                     for i in rows])


def lse_merge(parts):
    """Merge partial softmax results [(o_s, m_s, l_s)], each o_s unnormalised
    (sum_t e^{s_t - m_s} v_t), m_s the partial max and l_s = sum_t e^{s_t - m_s}:
    o = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s, M = max_s m_s.
    Used to pin that splitting the token range does not change the result."""
    M = max(m for _, m, _ in parts)
    num = sum(np.exp(m - M) * o for o, m, _ in parts)
    den = sum(np.exp(m - M) * l for _, m, l in parts)
    return num / den
