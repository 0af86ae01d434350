"""Mixed-precision group-wise quantized KV cache and decode attention for B200.

The compute lives in librq.so (CUDA, sm_100a) behind the C ABI of
include/rq.h; this package is its ctypes binding plus the synthetic workload
definitions.  Importing the package does not load the library; the first
call does, and fails loudly if it has not been built.
"""

from .api import (QuantizedKVCache, rq_allocate_bits, rq_cache_bytes, rq_cap_weights,  # noqa: F401
                  rq_fit_distortion, rq_measure_distortion)

__all__ = ["QuantizedKVCache", "rq_allocate_bits", "rq_cache_bytes", "rq_cap_weights", "rq_fit_distortion",
           "rq_measure_distortion"]
