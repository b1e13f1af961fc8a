"""Seeded synthetic workloads for the TokenGate gated-prefill path.

This package only draws random numbers and lays out shapes.  It holds none of
the method's arithmetic (no RMSNorm, no gate MLP, no selection, no softmax),
so both the CPU oracle and the CUDA path can take their inputs from it without
sharing any computation.
"""

from .configs import CONFIGS, Workload, get_config, masked_budgets  # noqa: F401
from .gen import (  # noqa: F401
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_attention_inputs,
    make_gate_inputs,
    make_gate_weights,
    make_scores,
)
