"""Seeded synthetic calibration inputs for CLHA (weight-shared MoE quantization).

This package only draws inputs: activations with a low-rank-plus-diagonal covariance, cross-layer
drift, router logits, outlier channels and expert weights, rounded to the storage dtype. It holds
none of the method's arithmetic (routing, Hessians, aggregation, factorisation, GPTQ, loss), so the
float64 oracle and the CUDA path can both read from it without sharing any computation.
"""
from .workloads import WORKLOADS, Workload, workload  # noqa: F401
