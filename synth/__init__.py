"""Seeded synthetic workloads for the head-wise sparse attention layer.

This package only draws inputs (random tensors, needle keys, ragged lengths).
It computes none of the layer's arithmetic (no indexer scores, no softmax, no
top-p, no RoPE, no attention), so both the CUDA path and the CPU oracle can
consume the same bytes without sharing any of the method's code.
"""

from .workloads import LayerShape, WORKLOADS, make_decode_inputs, make_prefill_inputs, workload

__all__ = ["LayerShape", "WORKLOADS", "make_decode_inputs", "make_prefill_inputs", "workload"]
