"""CPU oracle of the APB prefill path: test infrastructure, never the product.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this package.
"""
from .apb_oracle import (retaining_scores, retaining_scores_query_aware, compress_indices, passing_blocks,
                         host_attention, visible_pairs)

__all__ = ["retaining_scores", "retaining_scores_query_aware", "compress_indices", "passing_blocks",
           "host_attention", "visible_pairs"]
