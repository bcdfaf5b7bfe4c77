"""CPU binary64 oracle for exact fused linear cross-entropy.

Test infrastructure: imported only by the tests, the smoke check and the
benchmark's CPU-baseline leg.  It shares no code with the CUDA path.
"""
from .flce_oracle import (IGNORE_INDEX, backward, chunked, forward, forward_backward,
                          objective, row_outputs, row_scales, supervised_rows,
                          vocab_outputs)
from .flce_filtered import backward_filtered
from .flce_shards import shard_backward, shard_combine, shard_partials

__all__ = ["IGNORE_INDEX", "backward", "backward_filtered", "chunked", "forward", "forward_backward",
           "objective", "row_outputs", "row_scales", "shard_backward", "shard_combine",
           "shard_partials", "supervised_rows", "vocab_outputs"]
