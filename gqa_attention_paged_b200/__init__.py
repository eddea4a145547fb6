"""gqa_attention_paged_b200: grouped-query attention over a paged KV cache on B200.

The compute lives in libgqa_paged.so (hand-written sm_100a CUDA behind a C ABI, see
include/gqa_paged.h).  `gqa_attention_paged_b200.binding` marshals torch tensors into
that ABI; it loads the library on first use and raises if it is missing.  Importing this
package loads nothing.
"""

__all__ = ["binding", "inputs"]
