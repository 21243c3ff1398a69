"""Seeded synthetic workloads for the FlashLoop loop-r attention sublayer.

This package holds no arithmetic of the method: it only draws weights and
hidden states, rounds them to bf16 and describes the five workload shapes.
Both the CPU oracle and the CUDA path take their inputs from here.
"""
from .gen import (  # noqa: F401
    Config,
    CONFIGS,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    round_half_up,
    make_weights,
    make_hidden_states,
    make_decode_tokens,
)
