"""Seeded synthetic inputs for the MLA workloads (no attention arithmetic lives here)."""
from .configs import ORDER, TENSOR_IDS, WORKLOADS, Workload, lengths, make_inputs, make_weights, shrink

__all__ = ["ORDER", "TENSOR_IDS", "WORKLOADS", "Workload", "lengths", "make_inputs", "make_weights", "shrink"]
