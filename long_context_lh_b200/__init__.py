"""B200-native (sm_100a) hot path of one Lighthouse Attention layer.

`long_context_lh_b200.lighthouse` is the ctypes binding of the C-ABI library
(include/lighthouse.h); `long_context_lh_b200.synth` draws the seeded synthetic
inputs; `long_context_lh_b200.build` compiles the CUDA sources in-tree.
The binding is imported lazily so that the input generator and the build step
work on a host without the built library.
"""
__all__ = ["lighthouse", "synth", "build", "block"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
