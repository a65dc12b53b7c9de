"""CPU oracle for the asymmetric-precision quantized KV cache (KVSplit K8V4 and friends).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only the tests, the smoke check of the graft
entry point and the CPU-baseline leg of the benchmark do.  It shares no code,
tables or constants with the CUDA path; it is plain NumPy in float64 (with the
fp16 / fp32 roundings the storage format fixes) so that a reader can check it
against the source pages by eye.

Source pages (cited by title and section):
  * "KVSplit - contexto 2 a 3 vezes mais longo em Apple Silicon"
    (pt.news.hada.io/topic?id=20969): K and V at different bit widths, the
    per-configuration KV memory table, runtime quantisation of the cache,
    attention through the flash-attention path.
  * "KVBoost acelera inferencia de LLMs em 4,49x com cache reutilizavel"
    (omapapaper.com.br): corroborates int8 keys / int4 values.
  * "Reutilizacao de Cache KV para Conversas Longas no Apple Silicon"
    (openclawradar.com): keep the cache and process only the new tokens,
    which is what chunked prefill over a resident cache computes.

Every function is pinned by a test in tests/ against something other than
itself (the pages' printed byte table, exact rational arithmetic, closed-form
special cases, brute force); see each function's docstring for its pin.
"""
from .kvq_oracle import *  # noqa: F401,F403
