"""B200-native (sm_100a) inference forward pass of Hamming Attention Distillation.

The work happens in the CUDA library ``libhad.so`` behind the C ABI declared
in ``include/had.h``; ``had`` is its thin ctypes binding.  Importing the
package does not load the library; ``from sparse_attention_sigma_b200 import
had`` does, and fails loudly if it is missing.
"""
import importlib

__all__ = ["had"]


def __getattr__(name):
    if name == "had":
        return importlib.import_module(__name__ + ".had")
    raise AttributeError(name)
