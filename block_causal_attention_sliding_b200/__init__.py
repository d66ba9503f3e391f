"""Streaming block-causal sink + sliding-window attention for B200 (sm_100a)."""
from .configs import WORKLOADS, Workload  # noqa: F401
