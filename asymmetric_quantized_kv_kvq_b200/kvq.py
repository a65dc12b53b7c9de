"""Python binding of libkvq (include/kvq.h) through ctypes.

Argument marshalling only: torch tensors supply device pointers and the
current CUDA stream; every step of the computation runs in the library's
kernels.  If the library is missing the binding raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK = 0
STATUS_NAMES = {
    0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED", 3: "KVQ_ERR_OUT_OF_MEMORY",
    4: "KVQ_ERR_CAPACITY", 5: "KVQ_ERR_CUDA", 6: "KVQ_ERR_DEVICE_CHECK", 7: "KVQ_ERR_WORKSPACE",
}
KVQ_CACHE_HOST_ONLY = 1
KVQ_CACHE_DECODE_TENSOR_CORES = 2
KVQ_MAX_BATCH = 256
KVQ_NOALLOC_SCRATCH_BYTES = 8 << 20


class KvqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))


class CacheConfig(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32), ("page_tokens", ctypes.c_int32),
        ("max_seqs", ctypes.c_int32), ("flags", ctypes.c_int32), ("max_tokens", ctypes.c_int64),
        ("max_seq_tokens", ctypes.c_int64), ("layer_k_bits", ctypes.POINTER(ctypes.c_int32)),
        ("layer_v_bits", ctypes.POINTER(ctypes.c_int32)),
    ]


_i32, _i64, _u32, _f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float
_p, _sz = ctypes.c_void_p, ctypes.c_size_t
_pi32, _pi64, _psz, _pu32 = (ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64),
                            ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_uint32))

# name -> (restype, argtypes); the exported C ABI
SIGNATURES = {
    "kvq_footprint_bytes": (_i32, [ctypes.POINTER(CacheConfig), _i64, _pi64, _pi64]),
    "kvq_cache_create": (_i32, [ctypes.POINTER(CacheConfig), ctypes.POINTER(_p)]),
    "kvq_cache_destroy": (_i32, [_p]),
    "kvq_cache_footprint": (_i32, [_p, _pi64, _pi64, _pi64]),
    "kvq_seq_extend": (_i32, [_p, _i32, _pi32, _pi32, _p]),
    "kvq_seq_release": (_i32, [_p, _i32]),
    "kvq_seq_truncate": (_i32, [_p, _i32, _i64]),
    "kvq_seq_fork": (_i32, [_p, _i32, _i32, _i64, _p]),
    "kvq_seq_length": (_i32, [_p, _i32, _pi64]),
    "kvq_seq_set_window": (_i32, [_p, _i32, _i64]),
    "kvq_seq_page": (_i32, [_p, _i32, _i32, _pi32]),
    "kvq_append": (_i32, [_p, _i32, _i32, _pi32, _pi32, _p, _p, _p]),
    "kvq_decode_workspace_size": (_i32, [_p, _i32, _i32, _psz]),
    "kvq_decode_attn": (_i32, [_p, _i32, _i32, _pi32, _i32, _p, _p, _f32, _p, _sz, _p]),
    "kvq_decode_attn_noalloc": (_i32, [_p, _i32, _i32, _pi32, _i32, _p, _p, _f32, _p]),
    "kvq_decode_append_attn": (_i32, [_p, _i32, _i32, _pi32, _i32, _p, _p, _p, _p, _f32, _p, _sz, _p]),
    "kvq_decode_layers_workspace_size": (_i32, [_p, _i32, _i32, _i32, _psz]),
    "kvq_decode_attn_layers": (_i32, [_p, _i32, _i32, _i32, _pi32, _i32, _p, _p, _p, _p, _f32, _p, _sz, _p]),
    "kvq_prefill_workspace_size": (_i32, [_p, _i32, _pi32, _pi32, _i32, _psz]),
    "kvq_prefill_attn": (_i32, [_p, _i32, _i32, _pi32, _pi32, _i32, _p, _p, _f32, _p, _sz, _p]),
    "kvq_export": (_i32, [_p, _i32, _i32, _i64, _i64, _p, _p, _p, _p, _p]),
    "kvq_cache_check": (_i32, [_p, _p, _pu32]),
    "kvq_cache_dedup": (_i32, [_p, _p, _pi64]),
    "kvq_status_string": (ctypes.c_char_p, [_i32]),
    "kvq_last_error": (ctypes.c_char_p, []),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkvq.so (built by `python -m asymmetric_quantized_kv_kvq_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise KvqError(2, f"{path} is not built; run `python -m asymmetric_quantized_kv_kvq_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != KVQ_OK:
        raise KvqError(status, load_library().kvq_last_error().decode())


def _i32_array(xs: Sequence[int]):
    return (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dev_fp16(t, name: str, shape: Optional[tuple] = None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise KvqError(1, f"{name} must be a CUDA tensor")
    if t.dtype != torch.float16:
        raise KvqError(1, f"{name} must be float16")
    if not t.is_contiguous():
        raise KvqError(1, f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise KvqError(1, f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def make_config(n_layers, n_kv_heads, head_dim, k_bits, v_bits, max_seqs, max_tokens,
                page_tokens=256, max_seq_tokens=0, host_only=False, decode_tc=False,
                layer_bits: Optional[Sequence[tuple]] = None) -> CacheConfig:
    """layer_bits: optional [(k_bits, v_bits)] per layer, replacing k_bits / v_bits layer by layer."""
    flags = (KVQ_CACHE_HOST_ONLY if host_only else 0) | (KVQ_CACHE_DECODE_TENSOR_CORES if decode_tc else 0)
    cfg = CacheConfig(n_layers, n_kv_heads, head_dim, k_bits, v_bits, page_tokens, max_seqs,
                      flags, max_tokens, max_seq_tokens, None, None)
    if layer_bits is not None:
        if len(layer_bits) != n_layers:
            raise KvqError(1, f"layer_bits has {len(layer_bits)} entries for {n_layers} layers")
        cfg._lk = _i32_array([kb for kb, _ in layer_bits])      # kept alive with the config
        cfg._lv = _i32_array([vb for _, vb in layer_bits])
        cfg.layer_k_bits = ctypes.cast(cfg._lk, ctypes.POINTER(ctypes.c_int32))
        cfg.layer_v_bits = ctypes.cast(cfg._lv, ctypes.POINTER(ctypes.c_int32))
    return cfg


def footprint_bytes(n_layers, n_kv_heads, head_dim, k_bits, v_bits, n_tokens, page_tokens=256, layer_bits=None):
    """(allocated, used) bytes of one sequence of n_tokens (library closed form)."""
    cfg = make_config(n_layers, n_kv_heads, head_dim, k_bits, v_bits, 1, max(1, n_tokens), page_tokens,
                      layer_bits=layer_bits)
    a, u = ctypes.c_int64(), ctypes.c_int64()
    _check(load_library().kvq_footprint_bytes(ctypes.byref(cfg), n_tokens, ctypes.byref(a), ctypes.byref(u)))
    return a.value, u.value


class Cache:
    """A paged KV cache at (k_bits, v_bits) precision on the current CUDA device."""

    def __init__(self, n_layers: int, n_kv_heads: int, head_dim: int, k_bits: int, v_bits: int,
                 max_seqs: int, max_tokens: int, page_tokens: int = 256, max_seq_tokens: int = 0,
                 host_only: bool = False, decode_tc: bool = False, layer_bits: Optional[Sequence[tuple]] = None):
        """layer_bits: optional [(k_bits, v_bits)] per layer (per-layer precision); k_bits / v_bits
        then only name the default."""
        self._lib = load_library()
        self.cfg = make_config(n_layers, n_kv_heads, head_dim, k_bits, v_bits, max_seqs, max_tokens,
                               page_tokens, max_seq_tokens, host_only, decode_tc, layer_bits)
        self.n_layers, self.n_kv_heads, self.head_dim = n_layers, n_kv_heads, head_dim
        self.k_bits, self.v_bits = k_bits, v_bits
        self.layer_bits = [tuple(x) for x in layer_bits] if layer_bits is not None else [(k_bits, v_bits)] * n_layers
        self.host_only = host_only
        h = ctypes.c_void_p()
        _check(self._lib.kvq_cache_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self._h = h
        self._ws = None

    # -- lifetime
    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            st = self._lib.kvq_cache_destroy(self._h)
            self._h = None
            self._ws = None
            _check(st)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -- bookkeeping
    def footprint(self):
        p, m, u = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(self._lib.kvq_cache_footprint(self._h, ctypes.byref(p), ctypes.byref(m), ctypes.byref(u)))
        return p.value, m.value, u.value

    def extend(self, seq_ids: Sequence[int], n_new: Sequence[int], stream=None) -> None:
        s = None if self.host_only else _stream(stream)
        _check(self._lib.kvq_seq_extend(self._h, len(seq_ids), _i32_array(seq_ids), _i32_array(n_new), s))

    def release(self, seq_id: int) -> None:
        _check(self._lib.kvq_seq_release(self._h, seq_id))

    def truncate(self, seq_id: int, new_len: int) -> None:
        _check(self._lib.kvq_seq_truncate(self._h, seq_id, new_len))

    def fork(self, src: int, dst: int, n_tokens: Optional[int] = None, stream=None) -> None:
        """Empty sequence `dst` shares the first n_tokens (default: all) positions of `src`."""
        n = self.length(src) if n_tokens is None else n_tokens
        s = None if self.host_only else _stream(stream)
        _check(self._lib.kvq_seq_fork(self._h, src, dst, n, s))

    def set_window(self, seq_id: int, window_tokens: int) -> None:
        """Rotating window: empty sequence `seq_id` keeps (and attends to) only its last window_tokens."""
        _check(self._lib.kvq_seq_set_window(self._h, seq_id, window_tokens))

    def length(self, seq_id: int) -> int:
        n = ctypes.c_int64()
        _check(self._lib.kvq_seq_length(self._h, seq_id, ctypes.byref(n)))
        return n.value

    def page(self, seq_id: int, page: int) -> int:
        p = ctypes.c_int32()
        _check(self._lib.kvq_seq_page(self._h, seq_id, page, ctypes.byref(p)))
        return p.value

    # -- compute
    def append(self, layer: int, seq_ids: Sequence[int], n_new: Sequence[int], k, v, stream=None) -> None:
        total = int(sum(n_new))
        shape = (total, self.n_kv_heads, self.head_dim)
        kp = _dev_fp16(k, "k", shape) if total else None
        vp = _dev_fp16(v, "v", shape) if total else None
        _check(self._lib.kvq_append(self._h, layer, len(seq_ids), _i32_array(seq_ids), _i32_array(n_new),
                                    kp, vp, _stream(stream)))

    def decode_workspace_size(self, n_seqs: int, n_q_heads: int) -> int:
        n = ctypes.c_size_t()
        _check(self._lib.kvq_decode_workspace_size(self._h, n_seqs, n_q_heads, ctypes.byref(n)))
        return n.value

    def _workspace(self, nbytes: int, device):
        import torch
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self._ws

    def decode(self, layer: int, seq_ids: Sequence[int], q, out=None, softmax_scale: float = 0.0,
               workspace=None, stream=None):
        """q: fp16 [B, Hq, D] on the GPU -> out fp16 [B, Hq, D]."""
        import torch
        B = len(seq_ids)
        if q.dim() != 3 or q.shape[0] != B or q.shape[2] != self.head_dim:
            raise KvqError(1, f"q has shape {tuple(q.shape)}, expected [{B}, Hq, {self.head_dim}]")
        Hq = q.shape[1]
        _dev_fp16(q, "q")
        if out is None:
            out = torch.empty_like(q)
        _dev_fp16(out, "out", tuple(q.shape))
        need = self.decode_workspace_size(B, Hq)
        ws = workspace if workspace is not None else self._workspace(need, q.device)
        _check(self._lib.kvq_decode_attn(self._h, layer, B, _i32_array(seq_ids), Hq, q.data_ptr(),
                                         out.data_ptr(), softmax_scale, ws.data_ptr(),
                                         ws.numel() * ws.element_size(), _stream(stream)))
        return out

    def decode_append(self, layer: int, seq_ids: Sequence[int], q, k_new, v_new, out=None,
                      softmax_scale: float = 0.0, workspace=None, stream=None):
        """kvq_decode_append_attn: quantise k_new / v_new (fp16 [B, Hkv, D]) into position len - 1
        of each sequence, then decode q over positions 0 .. len - 1 (one launch for quantized caches)."""
        import torch
        B = len(seq_ids)
        if q.dim() != 3 or q.shape[0] != B or q.shape[2] != self.head_dim:
            raise KvqError(1, f"q has shape {tuple(q.shape)}, expected [{B}, Hq, {self.head_dim}]")
        Hq = q.shape[1]
        _dev_fp16(q, "q")
        kp = _dev_fp16(k_new, "k_new", (B, self.n_kv_heads, self.head_dim))
        vp = _dev_fp16(v_new, "v_new", (B, self.n_kv_heads, self.head_dim))
        if out is None:
            out = torch.empty_like(q)
        _dev_fp16(out, "out", tuple(q.shape))
        need = self.decode_workspace_size(B, Hq)
        ws = workspace if workspace is not None else self._workspace(need, q.device)
        _check(self._lib.kvq_decode_append_attn(self._h, layer, B, _i32_array(seq_ids), Hq, q.data_ptr(), kp, vp,
                                                out.data_ptr(), softmax_scale, ws.data_ptr(),
                                                ws.numel() * ws.element_size(), _stream(stream)))
        return out

    def decode_layers_workspace_size(self, n_layers: int, n_seqs: int, n_q_heads: int) -> int:
        n = ctypes.c_size_t()
        _check(self._lib.kvq_decode_layers_workspace_size(self._h, n_layers, n_seqs, n_q_heads, ctypes.byref(n)))
        return n.value

    def decode_layers(self, layer0: int, seq_ids: Sequence[int], q, k_new=None, v_new=None, out=None,
                      softmax_scale: float = 0.0, workspace=None, stream=None):
        """kvq_decode_attn_layers: one decode step over layers layer0 .. layer0 + NL - 1.
        q: fp16 [NL, B, Hq, D]; k_new / v_new: fp16 [NL, B, Hkv, D] (quantised into position
        len - 1 first) or both None -> out fp16 [NL, B, Hq, D]."""
        import torch
        B = len(seq_ids)
        if q.dim() != 4 or q.shape[1] != B or q.shape[3] != self.head_dim:
            raise KvqError(1, f"q has shape {tuple(q.shape)}, expected [layers, {B}, Hq, {self.head_dim}]")
        NL, Hq = q.shape[0], q.shape[2]
        _dev_fp16(q, "q")
        if (k_new is None) != (v_new is None):
            raise KvqError(1, "k_new and v_new must both be given or both be None")
        kp = _dev_fp16(k_new, "k_new", (NL, B, self.n_kv_heads, self.head_dim)) if k_new is not None else None
        vp = _dev_fp16(v_new, "v_new", (NL, B, self.n_kv_heads, self.head_dim)) if v_new is not None else None
        if out is None:
            out = torch.empty_like(q)
        _dev_fp16(out, "out", tuple(q.shape))
        need = self.decode_layers_workspace_size(NL, B, Hq)
        ws = workspace if workspace is not None else self._workspace(need, q.device)
        _check(self._lib.kvq_decode_attn_layers(self._h, layer0, NL, B, _i32_array(seq_ids), Hq, q.data_ptr(), kp,
                                                vp, out.data_ptr(), softmax_scale, ws.data_ptr(),
                                                ws.numel() * ws.element_size(), _stream(stream)))
        return out

    def decode_noalloc(self, layer: int, seq_ids: Sequence[int], q, out=None, softmax_scale: float = 0.0,
                       stream=None):
        """kvq_decode_attn_noalloc: same result as decode(), scratch in the library's fixed array."""
        import torch
        B = len(seq_ids)
        if q.dim() != 3 or q.shape[0] != B or q.shape[2] != self.head_dim:
            raise KvqError(1, f"q has shape {tuple(q.shape)}, expected [{B}, Hq, {self.head_dim}]")
        _dev_fp16(q, "q")
        if out is None:
            out = torch.empty_like(q)
        _dev_fp16(out, "out", tuple(q.shape))
        _check(self._lib.kvq_decode_attn_noalloc(self._h, layer, B, _i32_array(seq_ids), q.shape[1],
                                                 q.data_ptr(), out.data_ptr(), softmax_scale, _stream(stream)))
        return out

    def prefill_workspace_size(self, seq_ids: Sequence[int], q_lens: Sequence[int], n_q_heads: int) -> int:
        n = ctypes.c_size_t()
        _check(self._lib.kvq_prefill_workspace_size(self._h, len(seq_ids), _i32_array(seq_ids),
                                                    _i32_array(q_lens), n_q_heads, ctypes.byref(n)))
        return n.value

    def prefill(self, layer: int, seq_ids: Sequence[int], q_lens: Sequence[int], q, out=None,
                softmax_scale: float = 0.0, workspace=None, stream=None):
        """q: fp16 [sum(q_lens), Hq, D] -> out fp16, same shape."""
        import torch
        total = int(sum(q_lens))
        if q.dim() != 3 or q.shape[0] != total or q.shape[2] != self.head_dim:
            raise KvqError(1, f"q has shape {tuple(q.shape)}, expected [{total}, Hq, {self.head_dim}]")
        Hq = q.shape[1]
        _dev_fp16(q, "q")
        if out is None:
            out = torch.empty_like(q)
        _dev_fp16(out, "out", tuple(q.shape))
        need = self.prefill_workspace_size(seq_ids, q_lens, Hq)
        ws = workspace if workspace is not None else self._workspace(need, q.device)
        _check(self._lib.kvq_prefill_attn(self._h, layer, len(seq_ids), _i32_array(seq_ids),
                                          _i32_array(q_lens), Hq, q.data_ptr(), out.data_ptr(),
                                          softmax_scale, ws.data_ptr(), ws.numel() * ws.element_size(),
                                          _stream(stream)))
        return out

    def export(self, layer: int, seq_id: int, tok0: int, n_tok: int, stream=None, device="cuda"):
        """Canonical codes / scales of tokens [tok0, tok0 + n_tok): dict of device tensors."""
        import torch
        H, D = self.n_kv_heads, self.head_dim

        def codes(bits):
            if bits == 16:
                return torch.empty((n_tok, H, D), dtype=torch.float16, device=device)
            if bits == 8:
                return torch.empty((n_tok, H, D), dtype=torch.int8, device=device)
            return torch.empty((n_tok, H, D // 2), dtype=torch.uint8, device=device)

        kb, vb = self.layer_bits[layer]
        kc, vc = codes(kb), codes(vb)
        ks = torch.empty((n_tok, H, D // 32), dtype=torch.float16, device=device) if kb != 16 else None
        vs = torch.empty((n_tok, H, D // 32), dtype=torch.float16, device=device) if vb != 16 else None
        ptr = lambda t: None if t is None else t.data_ptr()
        _check(self._lib.kvq_export(self._h, layer, seq_id, tok0, n_tok, ptr(kc), ptr(ks), ptr(vc), ptr(vs),
                                    _stream(stream)))
        return {"k_codes": kc, "k_scales": ks, "v_codes": vc, "v_scales": vs}

    def dedup(self, stream=None) -> int:
        """kvq_cache_dedup: merge full pages with identical bytes; returns the pages freed."""
        n = ctypes.c_int64()
        _check(self._lib.kvq_cache_dedup(self._h, _stream(stream), ctypes.byref(n)))
        return n.value

    def check(self, stream=None) -> None:
        """Synchronise and raise on any earlier asynchronous or device-side error."""
        d = ctypes.c_uint32()
        _check(self._lib.kvq_cache_check(self._h, None if self.host_only else _stream(stream), ctypes.byref(d)))
