"""B200-native paged-KV decode attention.

The computation lives in the CUDA shared library built from ``csrc/``; this
package holds its thin ctypes binding (``binding``) and the seeded input
generators (``workloads``). Loading the binding fails loudly when the library
is missing: there is no CPU fallback.
"""

__all__ = ["binding", "workloads"]
