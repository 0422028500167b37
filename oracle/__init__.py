"""fp64 CPU oracle for exact attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  It shares no code with the CUDA library.
"""
from . import philox  # noqa: F401
from .attention import (  # noqa: F401
    attention_backward,
    attention_decode,
    attention_forward,
    causal_visible,
    decode_split_combine,
    head_backward,
    head_backward_rows,
    head_forward,
    head_probs,
    tiled_softmax_then_matmul,
)
