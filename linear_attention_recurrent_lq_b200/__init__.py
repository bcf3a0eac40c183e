"""B200-native LeapQuant decode path: low-bit per-window recurrent state for
Gated DeltaNet / Kimi Delta Attention heads.

The compute lives in ``libleapquant.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in include/leapquant.h).  ``binding`` marshals torch tensors
into that ABI; ``inputs`` draws the seeded synthetic workloads.  Submodules
are imported on demand so that drawing inputs never loads the CUDA library.
"""
__all__ = ["binding", "inputs"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
