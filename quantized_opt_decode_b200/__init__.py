"""quantized_opt_decode_b200: group-wise 4-bit OPT-style decoding on one B200.

The hot path lives in libflexq.so (hand-written sm_100a CUDA behind the C ABI
of include/flexq.h).  ``flexq`` is its ctypes binding; ``device_model`` holds
the torch-side plumbing that allocates a synthetic model and its KV caches in
device memory and fills them through the library.  ``build`` compiles the
library, so importing the package does not load it: the binding is loaded on
first use and fails loudly when libflexq.so is missing.
"""

__all__ = ["flexq"]


def __getattr__(name):
    if name == "flexq":
        import importlib
        return importlib.import_module(__name__ + ".flexq")
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
