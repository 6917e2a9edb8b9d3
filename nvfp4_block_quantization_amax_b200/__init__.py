"""NVFP4 block quantization and block-scaled FP4 GEMM for B200 (sm_100a).

The compute lives in ``libnvfp4.so`` (hand-written CUDA behind a C ABI,
declared in ``include/nvfp4.h``).  The Python side only marshals arguments:
``api`` wraps the C entry points for torch tensors, ``synthetic`` draws seeded
inputs.  Nothing here falls back to a CPU implementation: if the library is
missing, the first call raises.
"""
__all__ = ["api", "synthetic"]


def __getattr__(name):
    if name in ("api", "synthetic", "_lib", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
