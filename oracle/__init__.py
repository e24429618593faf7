"""fp64 CPU oracle for exact attention (forward and backward).

TEST INFRASTRUCTURE ONLY. This package is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``, and by
nothing else. The product path (``exact_io_aware_66_b200``) never imports it, and
it imports nothing from the product path: the two share no code. The seeded input
generators that feed both live in ``exact_io_aware_66_b200/workloads.py`` and hold
none of the method's arithmetic.

Every function here is pinned by ``tests/test_oracle.py`` to closed forms,
invariants, brute force, finite differences and the pages' online-softmax
recurrence; none is "parity unpinned".
"""

from .attention import (  # noqa: F401
    attention_backward,
    attention_forward,
    attention_keys,
    attention_probabilities,
    attention_rows,
    online_softmax_stats,
    tiled_attention_forward,
)
from .dropout import dropout_keep, dropout_p8, keep_scale, philox4x32_10  # noqa: F401
from .fp8 import attention_forward_fp8, e4m3_decode  # noqa: F401
