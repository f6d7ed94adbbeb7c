"""Float64 CPU oracle (test infrastructure only; see oracle/attention.py)."""

from .attention import (  # noqa: F401
    allowed_keys,
    attention,
    attention_rows,
    online_attention_equations,
    online_attention_flowchart,
    scores,
    two_pass_softmax,
)
