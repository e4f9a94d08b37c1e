"""B200-native speculative-decoding verification sampler.

The compute path is ``libspecverify.so`` (hand-written sm_100a CUDA kernels
behind a C ABI, declared in ``include/specverify.h``).  ``binding`` marshals
torch device buffers into that ABI; ``workloads`` draws seeded synthetic
inputs.  Importing this package does not load the CUDA library; the first
call through ``binding`` does, and fails loudly if it is missing.
"""
__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
