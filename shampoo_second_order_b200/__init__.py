"""B200-native Shampoo optimizer step: a C-ABI CUDA library and its thin
Python binding.

Importing the package loads nothing; ``shampoo_second_order_b200.lib()``
loads the compiled library and raises if it is missing.
"""
