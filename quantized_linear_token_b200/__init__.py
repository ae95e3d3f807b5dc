"""OrbitQuant quantized linear layer for B200 (sm_100a).

The compute path is the C-ABI library ``liborbitquant.so`` (hand-written CUDA
kernels); ``binding`` marshals torch tensors into its calls.  Attributes of the
binding are resolved on first use, so importing ``workloads`` needs no GPU and
no built library.
"""

import importlib

__version__ = "0.1.0"

_SUBMODULES = {"binding", "workloads", "build"}


def __getattr__(name):
    if name.startswith("_") or name in _SUBMODULES:
        raise AttributeError(name)
    binding = importlib.import_module(__name__ + ".binding")
    return getattr(binding, name)
