"""Exact IO-aware attention (forward and backward) for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libfa_b200.so`` built from ``csrc/``;
the functions exported here only marshal arguments to it (see ``api.py``).
"""

from .inputs import WORKLOADS, Workload, make_inputs, make_qkv, workload  # noqa: F401
