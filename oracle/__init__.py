"""The oracle: a plain, slow, float64 CPU restatement of blockwise attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py``; never by the product
library or its Python binding, and it imports nothing from them.
"""

from .blockwise import attention, attention_rows, chunked_attention, merge

__all__ = ["attention", "attention_rows", "chunked_attention", "merge"]
