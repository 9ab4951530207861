"""CPU float64 oracle for the DSA hot path (test infrastructure only; see dsa_oracle)."""
from .dsa_oracle import (  # noqa: F401
    GATE_MODES,
    RELU_MODES,
    apply_gate,
    dsa_forward,
    index_scores,
    sparse_attention,
    topk_indices,
    window_attention,
)
