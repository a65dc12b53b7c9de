"""Seeded synthetic workloads and input generators.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds no arithmetic of the method (no quantisation, no
attention): only shapes, seeds and random fp16 tensors.

Workload shapes follow the KVSplit page (pt.news.hada.io, "KVSplit - contexto 2
a 3 vezes mais longo em Apple Silicon"): its memory table is quoted for a
22-layer model with 4 KV heads of width 64 (TinyLlama-shaped), and the larger
decode / prefill shapes are Llama-3-8B-like and 70B-like attention layers.
Values are ~N(0, 1) in fp16; a seeded subset of key channels is scaled x10 to
model the outlier channels that make keys the quantisation-sensitive half
(section "Assimetria entre key e value").

Every tensor is drawn by torch's generator from a seed derived from
(workload, tensor kind, layer, sequence, chunk); a token range of a sequence is
always the concatenation of fixed 4096-token chunks, so any slice can be
regenerated on its own.
"""
from __future__ import annotations

import dataclasses
import functools
from typing import Optional, Sequence

import torch

GEN_CHUNK = 4096          # tokens per independently seeded chunk
OUTLIER_SCALE = 10.0      # key outlier channels are scaled by this factor

_KINDS = {"k": 1, "v": 2, "q": 3, "outlier": 4, "lens": 5, "qchunk": 6}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    batch: int
    cached: int                      # cached tokens per sequence (decode)
    precisions: tuple                # e.g. ("K8V4",) or ("FP16", "K8V8", ...)
    outliers_per_head: int = 0       # key outlier channels per (layer, kv head)
    outlier_frac: float = 0.0        # or: fraction of all Hkv*D key channels per layer
    chunk: int = 0                   # prefill: tokens appended per sequence
    cached_lo: int = 0               # prefill: cached lengths ~ U{lo..hi}
    cached_hi: int = 0
    seed: int = 0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    # single attention layer, TinyLlama-shaped, 128 cached tokens
    "tinyllama-1l-128": Workload("tinyllama-1l-128", 1, 32, 4, 64, 1, 128, ("K8V4",),
                                 outliers_per_head=4),
    # full 22-layer TinyLlama-shaped cache at 8192 tokens, four precisions
    "tinyllama-22l-8k": Workload("tinyllama-22l-8k", 22, 32, 4, 64, 1, 8192,
                                 ("FP16", "K8V8", "K8V4", "K4V4"), outliers_per_head=4),
    # batched decode, Llama-3-8B-shaped attention
    "llama3-8b-b32-32k": Workload("llama3-8b-b32-32k", 32, 32, 8, 128, 32, 32768, ("K8V4",),
                                  outlier_frac=0.01),
    # long-context single sequence, 70B-shaped attention
    "llama70b-b1-128k": Workload("llama70b-b1-128k", 80, 64, 8, 128, 1, 131072,
                                 ("K8V4", "FP16"), outlier_frac=0.01),
    # ragged chunked prefill on a paged cache
    "prefill-16x4096": Workload("prefill-16x4096", 1, 32, 8, 128, 16, 0, ("K8V4",),
                                outlier_frac=0.01, chunk=4096, cached_lo=1024, cached_hi=65536),
}


def seed_for(*idx: int) -> int:
    """Deterministic 63-bit seed from a tuple of small non-negative ints
    (splitmix64 mixing; independent of Python's hash randomisation)."""
    m = (1 << 64) - 1
    h = 0x243F6A8885A308D3
    for v in idx:
        h = (h ^ (int(v) & m)) & m
        h = (h + 0x9E3779B97F4A7C15) & m
        z = h
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
        h = z ^ (z >> 31)
    return h & ((1 << 63) - 1)


def _wl_id(wl: Workload) -> int:
    return seed_for(sum(ord(c) * (i + 1) for i, c in enumerate(wl.name)), wl.seed)


def _randn(shape, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


@functools.lru_cache(maxsize=512)
def outlier_channels(wl: Workload, layer: int) -> torch.Tensor:
    """Boolean mask [Hkv, D] of key channels scaled by OUTLIER_SCALE in `layer`."""
    H, D = wl.n_kv_heads, wl.head_dim
    g = torch.Generator(device="cpu")
    g.manual_seed(seed_for(_wl_id(wl), _KINDS["outlier"], layer))
    mask = torch.zeros(H, D, dtype=torch.bool)
    if wl.outliers_per_head:
        for h in range(H):
            idx = torch.randperm(D, generator=g)[: wl.outliers_per_head]
            mask[h, idx] = True
    elif wl.outlier_frac:
        n = int(round(wl.outlier_frac * H * D))
        idx = torch.randperm(H * D, generator=g)[:n]
        mask.view(-1)[idx] = True
    return mask


@functools.lru_cache(maxsize=512)
def _outlier_mask_on(wl: Workload, layer: int, device: str) -> torch.Tensor:
    return outlier_channels(wl, layer).to(device)


def _chunk(wl: Workload, kind: str, layer: int, seq: int, c: int, device) -> torch.Tensor:
    x = _randn((GEN_CHUNK, wl.n_kv_heads, wl.head_dim),
               seed_for(_wl_id(wl), _KINDS[kind], layer, seq, c), device)
    if kind == "k":
        mask = _outlier_mask_on(wl, layer, str(device))
        x = torch.where(mask, x * OUTLIER_SCALE, x)
    return x.to(torch.float16)


def gen_kv(wl: Workload, layer: int, seq: int, tok0: int, n: int,
           device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """fp16 K and V of tokens [tok0, tok0+n) of sequence `seq` in `layer`,
    each [n, Hkv, D] (token-major, as a QKV projection writes them)."""
    ks, vs = [], []
    t = tok0
    while t < tok0 + n:
        c = t // GEN_CHUNK
        lo = t - c * GEN_CHUNK
        hi = min(GEN_CHUNK, tok0 + n - c * GEN_CHUNK)
        ks.append(_chunk(wl, "k", layer, seq, c, device)[lo:hi])
        vs.append(_chunk(wl, "v", layer, seq, c, device)[lo:hi])
        t = c * GEN_CHUNK + hi
    if not ks:
        z = torch.empty((0, wl.n_kv_heads, wl.head_dim), dtype=torch.float16, device=device)
        return z, z.clone()
    return torch.cat(ks), torch.cat(vs)


def gen_q(wl: Workload, layer: int, step: int, n_seqs: Optional[int] = None,
          device="cpu") -> torch.Tensor:
    """Decode queries for one step: fp16 [B, Hq, D] ~ N(0, 1)."""
    B = wl.batch if n_seqs is None else n_seqs
    x = _randn((B, wl.n_q_heads, wl.head_dim),
               seed_for(_wl_id(wl), _KINDS["q"], layer, step), device)
    return x.to(torch.float16)


def gen_q_chunk(wl: Workload, layer: int, seq: int, n: int, device="cpu") -> torch.Tensor:
    """Prefill queries of one sequence's chunk: fp16 [n, Hq, D] ~ N(0, 1)."""
    x = _randn((n, wl.n_q_heads, wl.head_dim),
               seed_for(_wl_id(wl), _KINDS["qchunk"], layer, seq), device)
    return x.to(torch.float16)


def cached_lengths(wl: Workload, n_seqs: Optional[int] = None) -> list:
    """Prefill workloads: seeded cached lengths, uniform integers in
    [cached_lo, cached_hi]; decode workloads: `cached` for every sequence."""
    B = wl.batch if n_seqs is None else n_seqs
    if not wl.cached_hi:
        return [wl.cached] * B
    g = torch.Generator(device="cpu")
    g.manual_seed(seed_for(_wl_id(wl), _KINDS["lens"]))
    return torch.randint(wl.cached_lo, wl.cached_hi + 1, (B,), generator=g).tolist()


def random_fp16(shape: Sequence[int], seed: int, scale: float = 1.0, device="cpu") -> torch.Tensor:
    """Generic seeded fp16 ~ N(0, scale^2) tensor for edge-case tests."""
    x = _randn(tuple(shape), seed_for(seed, 0x5EED), device)
    return (x * scale).to(torch.float16)


def parse_precision(name: str) -> tuple:
    """'K8V4' -> (8, 4); 'FP16' -> (16, 16)."""
    if name.upper() == "FP16":
        return 16, 16
    n = name.upper()
    assert n[0] == "K" and "V" in n, name
    kb, vb = n[1:].split("V")
    return int(kb), int(vb)
