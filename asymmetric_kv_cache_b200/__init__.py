"""asymmetric_kv_cache_b200: decode attention over an asymmetrically quantized
KV cache (keys per channel, values per token, fp16 tail) for NVIDIA B200.

The compute path lives in the CUDA library ``libkvq.so`` (``csrc/``); the
Python side in ``kvq.py`` only marshals arguments for its C ABI.  Import
``asymmetric_kv_cache_b200.kvq`` explicitly; this package module is kept free
of side effects so that the seeded input generators in ``inputs.py`` can be
imported without loading the library.
"""
