"""fp64 CPU oracle for causal scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product path (the
CUDA library and its binding) never does.  It shares no code with the CUDA path.
"""
from .attention import attention, build, library_path, num_cores, rope_append, widen_bits
from .backward import attention_backward
from .paged import gather_pages, paged_attention

__all__ = ["attention", "attention_backward", "build", "gather_pages", "library_path", "num_cores", "paged_attention",
           "rope_append", "widen_bits"]
