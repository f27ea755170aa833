"""fp64 CPU oracle of the Shampoo optimizer step.

Test infrastructure only: used by the tests, the smoke check and the bench's
CPU baseline / reference leg.  The product (``shampoo_second_order_b200``)
never imports it, and it imports nothing from the product.
"""
from .shampoo_oracle import (  # noqa: F401
    GRAFT_ADAGRAD, GRAFT_NONE, SIDE_LEFT, SIDE_RIGHT, SIDES_BOTH, ShampooOracle, block_partition,
    coupled_newton_inverse_root, inverse_root, vector_segments)
