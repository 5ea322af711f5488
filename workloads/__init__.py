"""Seeded synthetic workloads: sizes (``configs``) and input bytes (``synth``)."""
from .configs import HEADLINE, ORDER, WORKLOADS, Workload, get, scaled
from .synth import Inputs, bf16_bits_to_f32, f32_to_bf16_bits, make_inputs

__all__ = ["HEADLINE", "ORDER", "WORKLOADS", "Workload", "get", "scaled", "Inputs",
           "bf16_bits_to_f32", "f32_to_bf16_bits", "make_inputs"]
