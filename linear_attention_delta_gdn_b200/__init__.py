"""B200-native Gated Delta Rule-2 operator (Gated DeltaNet-2), sm_100a.

The operator runs in ``libgdn2.so`` (C ABI in ``include/gdn2.h``); this package
holds its CUDA sources (``csrc/``), the in-tree build script (:mod:`.build`),
the ctypes binding (:mod:`.binding`) and the seeded synthetic-input generator
(:mod:`.inputs`). Importing the package does not load the library; the binding
loads it on first use and raises if it is missing.
"""

__all__ = ["gdn2_fwd", "gdn2_bwd", "gdn2_decode_step", "gdn2_workspace_size", "gated_delta_rule2",
           "GatedDeltaRule2", "Gdn2Error"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
