"""CPU float64 oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline /
reference arm may import this package.  The CUDA library never does.
"""
from .attention import attention_backward, attention_forward, default_scale
from .tiled_model import (flash_forward_tiled, merge, running_stats,
                          sum_of_block_outputs)

__all__ = [
    "attention_forward", "attention_backward", "default_scale",
    "flash_forward_tiled", "merge", "running_stats", "sum_of_block_outputs",
]
