"""B200-native chunkwise gated linear attention (forward and backward).

The compute path is the CUDA library libgla_b200.so (C ABI in include/gla.h); the
Python entry points below only marshal torch tensors into it. Importing the entry
points loads the library and raises if it has not been built.
"""
__version__ = "0.1.0"


def __getattr__(name):
    # Lazy: `linear_rnn_b200.inputs` and `.build` import without loading the library.
    if name in ("gla_fwd", "gla_bwd", "gla_workspace_bytes", "gla_check_device_status", "make_problem"):
        from . import ops
        return getattr(ops, name)
    if name in ("GlaError",):
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
