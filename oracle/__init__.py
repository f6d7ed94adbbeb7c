"""Float64 CPU oracle (test infrastructure only; see oracle/attention.py)."""

from .attention import (  # noqa: F401
    allowed_keys,
    attention,
    attention_backward,
    attention_key_range,
    attention_rows,
    merge_splits,
    online_attention_equations,
    online_attention_flowchart,
    scores,
    split_kv_attention,
    two_pass_softmax,
)
