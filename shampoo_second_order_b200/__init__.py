"""B200-native Shampoo optimizer step: a C-ABI CUDA library and its thin
Python binding.

Importing the package loads nothing; ``lib()`` loads the compiled library and
raises if it is missing.  ``Shampoo`` (in ``optimizer``) wraps one library
context for torch tensors.
"""
from ._lib import lib  # noqa: F401


def __getattr__(name):
    if name in ("Shampoo", "batched_inverse_root"):
        from . import optimizer
        return getattr(optimizer, name)
    raise AttributeError(name)
