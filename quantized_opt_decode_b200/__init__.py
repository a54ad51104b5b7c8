"""quantized_opt_decode_b200: group-wise 4-bit OPT-style decoding on one B200.

The hot path lives in libflexq.so (hand-written sm_100a CUDA behind the C ABI
of include/flexq.h).  ``flexq`` is its ctypes binding; ``device_model`` holds
the torch-side plumbing that allocates a synthetic model and its KV caches in
device memory and fills them through the library.
"""
from . import flexq  # noqa: F401  (fails loudly when libflexq.so is missing)

__all__ = ["flexq"]
