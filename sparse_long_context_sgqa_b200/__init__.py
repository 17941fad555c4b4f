"""Sparse GQA global-attention hot path for B200 (sm_100a).

The compute path is the CUDA library ``libsgqa.so`` (C ABI in
``include/sgqa.h``); ``sparse_long_context_sgqa_b200.binding`` marshals torch
tensors to it.  There is no CPU fallback: importing the binding fails if the
library is missing.
"""
from .inputs import WORKLOADS, Workload  # noqa: F401
