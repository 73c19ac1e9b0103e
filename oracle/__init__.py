"""CPU fp64 oracle for exact attention (TEST INFRASTRUCTURE ONLY).

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``.  It shares no code with the CUDA path and imports nothing
from it.  See ``oracle/attention.py`` for the definitions and their sources.
"""

from .attention import (  # noqa: F401
    backward,
    backward_head,
    blocked_forward_head,
    decode_paged,
    forward,
    forward_head,
    forward_rows_head,
    hidden_keys,
    kv_head,
    paged_rows,
    probs_head,
    scores_head,
)
