"""kvq: B200-native quantized-KV decode attention with a certified error bound.

The compute path is the CUDA library ``libkvq.so`` (built from ``csrc/``),
reached through the thin ctypes binding ``quantized_decode_attention_kvq_b200.kvq``.
``inputs`` holds the seeded synthetic workloads.  Importing the package does
not load the library; ``kvq`` raises if the library is missing.
"""

__all__ = ["inputs", "kvq"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
