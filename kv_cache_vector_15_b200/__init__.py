"""TurboQuant KV-cache / vector quantization hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libtq.so`` (hand-written CUDA behind a C ABI, see
``include/tq.h``); ``kv_cache_vector_15_b200.tq`` is its thin ctypes binding.
``kv_cache_vector_15_b200.inputs`` draws the seeded synthetic workloads.
"""
