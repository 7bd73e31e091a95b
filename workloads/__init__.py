"""Seeded synthetic workloads for the LLaTTE sequence-module forward pass.

This package only describes shapes and draws random numbers. It holds none of
the method's arithmetic, so both the fp64 oracle and the CUDA path can consume
its output without sharing any computation.
"""
from .configs import Dims, Workload, WORKLOADS, workload
from .gen import Inputs, make_inputs, make_event_ages, draw_lengths, draw_weights, round_to_bf16

__all__ = ["Dims", "Workload", "WORKLOADS", "workload", "Inputs", "make_inputs", "make_event_ages",
           "draw_lengths", "draw_weights", "round_to_bf16"]
