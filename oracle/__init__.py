"""fp64 CPU oracle for the STILL hybrid-attention layer -- TEST INFRASTRUCTURE.

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline leg
(and its `--impl reference` arm) may import this package.  It shares no code
with the CUDA library: `still_oracle.c` is a separate, plain C implementation
written from the definitions ("STILL: Selecting Tokens for Intra-Layer Hybrid
Attention to Linearize LLMs"), and `brute.py` is a second, pure numpy one for
tiny inputs.
"""
from .oracle import (  # noqa: F401
    Dims,
    build,
    saliency,
    diagonal_score,
    topk,
    npmap,
    prefill,
    linear_state,
    Decoder,
)
