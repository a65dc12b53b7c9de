"""Asymmetric-precision quantized KV cache (K8V4, K8V8, K4V4, K4V8, FP16) for B200.

The product is the C-ABI library libkvq.so (include/kvq.h); the submodule
`kvq` is its thin ctypes binding (importing it does not load the library;
the first call does).  `inputs` holds the seeded synthetic workloads.
"""
