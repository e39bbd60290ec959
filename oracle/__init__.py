"""CPU oracle for the TokenGate gated-prefill path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The product path never does.
"""
from .tg_oracle import (  # noqa: F401
    gate_scores, gate_value, gelu, gather, gated_attention, gated_attention_weights,
    kept_count, prefill_above_L, prefill_from_scores, topk_select,
)
