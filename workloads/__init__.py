"""Seeded synthetic workloads for the MHA2MLA latent-cache decode path.

This package holds only shapes and random inputs: the synthetic MHA layer
(W_q, W_k, W_v), its calibration and decode activations, the context tokens and
the sequence lengths. It contains none of the method's arithmetic (no pair
scoring, no SVD, no RoPE, no attention), so that the CPU oracle and the CUDA
path can both draw their inputs from it without sharing any computation.
"""

from .configs import WORKLOADS, PARITY_WORKLOADS, EXTRA_WORKLOADS, Workload, get  # noqa: F401
from . import generate  # noqa: F401
