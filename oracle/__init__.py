"""fp64 CPU oracle for paged-KV decode attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this package. The product path (the CUDA library and
its binding) never imports, links or runs it.
"""

from .oracle import (  # noqa: F401
    build,
    e4m3_to_double,
    bf16_to_double,
    paged_decode_attn,
    merge_states,
    ORACLE_KV_BF16,
    ORACLE_KV_FP8_E4M3,
    CAUSAL_OFF,
    CAUSAL_BOTTOM_RIGHT,
)
