"""B200 (sm_100a) attention hot path for encoder context: paged cross-attention over a
context written once, and cacheless ragged attention over the spans of one packed forward.

The work runs in the C-ABI library ``librae.so`` (include/rae.h); this package is its thin
Python binding.  Importing the package does not load the library; constructing a Context
does, and fails loudly when the library has not been built.
"""
from .api import (  # noqa: F401
    Context,
    CrossAttention,
    Plan,
    RaeError,
    RaggedAttention,
    plan_paged_host,
    plan_ragged_host,
)
