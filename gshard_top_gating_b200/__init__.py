"""GShard top-k Mixture-of-Experts layer forward on one B200 (sm_100a).

The computation lives in the CUDA library `libgshard_moe.so` (C ABI in
include/moe.h).  `_lib` is the ctypes binding with the C entry points' names,
`layer.MoeLayer` an owning wrapper, `inputs` the seeded synthetic workloads.
Importing this package does not load the library; `_lib` does, and fails
loudly if it has not been built.
"""

__all__ = ["MoeLayer"]


def __getattr__(name):
    if name == "MoeLayer":
        from .layer import MoeLayer
        return MoeLayer
    raise AttributeError(name)
