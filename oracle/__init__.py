"""CPU float64 oracle for exact softmax attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The CUDA library never imports,
links or calls it, and it never imports the CUDA library.
"""

from .attention_ref import (  # noqa: F401
    BLOCK,
    attention_backward,
    attention_backward_gqa,
    attention_forward,
    attention_forward_gqa,
    gqa_expand,
    gqa_reduce,
    dropout_keep,
    dropout_scale,
    dropout_threshold,
    head_backward,
    head_backward_block,
    head_backward_cols,
    head_backward_rows,
    head_forward_rows,
    merge_partials,
    safe_softmax,
    valid_mask,
)
from .philox_ref import philox4x32_10, philox_block, weyl_constants  # noqa: F401
from .projection_ref import qkv_projection  # noqa: F401
from .varlen_ref import attention_backward_varlen, attention_forward_varlen  # noqa: F401
