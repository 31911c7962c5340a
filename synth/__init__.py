"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This package draws random data only: it holds none of the codec or attention
arithmetic (no assignment, projection, quantisation, decode or softmax).
"""
from .gen import WORKLOADS, Workload, make_codec, make_tokens, make_problem  # noqa: F401
