"""Block-scaled GEMM D = A * B^T for one NVIDIA B200 (sm_100a).

The computation runs in the CUDA library ``libbsp.so`` (C ABI in ``include/bsp.h``);
this package is its thin Python binding.  There is no CPU fallback: a call without the
built library or without a B200 raises.
"""

__all__ = ["ops", "lib", "shard"]


def __getattr__(name):
    if name in ("ops", "lib", "shard"):
        import importlib

        return importlib.import_module(f".{'_lib' if name == 'lib' else name}", __name__)
    raise AttributeError(name)
