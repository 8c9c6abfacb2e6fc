"""CPU fp64 oracle for exact scaled dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``exact_io_aware_91_b200``) never imports it, and this
package imports nothing from the product: the two share no code.

The oracle materialises the full N x N score and probability matrices on the host
in float64 -- exactly what the IO-aware method avoids -- so that a reader can check
it against the definition by eye.
"""

from .attention import (  # noqa: F401
    attention_probs,
    attention_forward,
    attention_forward_rows,
    attention_backward_dq_rows,
    attention_backward,
    online_softmax_forward,
    loop_attention_forward,
    loop_attention_backward,
    kv_head_of,
    attention_forward_gqa,
    attention_backward_gqa,
    apply_window,
)
from .fp8 import e4m3_decode, attention_forward_fp8, attention_forward_fp8_rows  # noqa: F401
