"""Float64 CPU oracle (test infrastructure only; see ``oracle.attention``).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .attention import (  # noqa: F401
    allowed_mask,
    attention_backward,
    attention_forward,
    attention_forward_offset,
    attention_forward_rows,
    attention_probabilities,
    attention_scores,
    decode_forward,
    decode_paged_forward,
    default_scale,
    merge_partials,
    online_softmax_forward,
)
