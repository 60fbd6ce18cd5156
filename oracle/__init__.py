"""CPU oracle of the RoM projection block (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference arm may import this package. The product path never does.
"""
from .rom_oracle import (block_backward, block_forward, causal_conv1d, dispatch, inproj_forward,
                         route, selective_scan, sigmoid, silu, silu_grad, softmax, softplus,
                         ssm_core, variant_block_forward)

__all__ = ["block_backward", "block_forward", "causal_conv1d", "dispatch", "inproj_forward",
           "route", "selective_scan", "sigmoid", "silu", "silu_grad", "softmax", "softplus",
           "ssm_core", "variant_block_forward"]
