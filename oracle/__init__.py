"""fp64 CPU oracle for prefix-masked attention forward.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path never imports this package,
and this package never imports the product.
"""
from .oracle import (  # noqa: F401
    build_oracle,
    attn_prefix,
    attn_chunk,
    attn_segments,
    attn_masked,
    lse_combine,
    num_threads,
    set_num_threads,
)
