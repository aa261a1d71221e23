"""Seeded synthetic workloads for the loss-scaled FP32-master step.

This module is shared by the tests, the benchmark and the oracle harness.  It
holds none of the step's arithmetic: it only describes parameter lists
(tensor shapes, master-weight initialisation, gradient laws, hyperparameters)
and draws seeded inputs from them with integer hashing and table look-ups.
FP16 gradients are produced directly as binary16 bit patterns (no float ->
half conversion is involved), so that neither side of a parity test shares a
rounding routine with the generator.

Workloads (sizes in parameters):
  flat1m         1 flat tensor, 1 048 576
  resnet50       161 tensors, 25 557 032 (ResNet-50 conv/BN/FC shapes)
  gpt2_medium    292 tensors, 354 823 168 (24 layers, d=1024, vocab 50257)
  gpt_1p3b       292 tensors, 1 315 723 264 (24 layers, d=2048, FFN 8192)
  ragged20k      20 000 tensors, sizes floor(exp(U[0, ln 2^20))), seeded
"""
from .configs import CONFIGS, Config, TensorSpec, get  # noqa: F401
from .gen import (GradLayout, cdf_table, fp16_magnitude_values, make_grads,  # noqa: F401
                  make_master, uniform_u32)
