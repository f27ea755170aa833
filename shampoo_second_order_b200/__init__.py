"""B200-native Shampoo optimizer step: a C-ABI CUDA library and its thin
Python binding.

Importing the package loads nothing; ``lib()`` loads the compiled library and
raises if it is missing.  ``Shampoo`` (in ``optimizer``) wraps one library
context for torch tensors; ``ShardedShampoo`` (in ``sharded``) splits the
parameters of a data-parallel job over ranks by owner.
"""
from ._lib import lib  # noqa: F401


def __getattr__(name):
    if name in ("Shampoo", "batched_inverse_root"):
        from . import optimizer
        return getattr(optimizer, name)
    if name == "ShardedShampoo":
        from .sharded import ShardedShampoo
        return ShardedShampoo
    raise AttributeError(name)
