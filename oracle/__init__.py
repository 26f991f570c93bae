"""CPU oracle for the attention hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  The product (the CUDA library and its Python binding) never
imports it, and this package imports nothing from the product: the two share no
kernels, helpers, tables or pre/post-processing.  Inputs come from the seeded
generators in ``ragged_attention_encoder_b200.inputs``, which hold no attention
arithmetic.

Everything here is plain float64 NumPy, written for a reader to check by eye against
the definitions it follows (see ``attention.py``).  Every function is pinned by
``tests/test_oracle.py`` to results fixed by mathematics or by an independent library
routine (closed forms, invariants, brute-force enumeration, and
``torch.nn.functional.scaled_dot_product_attention`` in float64).  No function here is
"parity unpinned".
"""
from .attention import (  # noqa: F401
    append_kv,
    as_f64,
    attention_rows,
    block_causal_visible,
    causal_append_visible,
    context_write,
    gather_paged_kv,
    merge_partials,
    paged_causal_attention,
    paged_causal_attention_rows,
    paged_cross_attention,
    paged_cross_attention_rows,
    partial_attention_with_lse,
    project_kv,
    ragged_block_causal_attention,
    ragged_block_causal_rows,
    ragged_cross_attention,
)
