"""Seeded synthetic inputs for the SSD scan: shared by the tests, the bench and the oracle.

Holds random-number generation and the workload table only; none of the scan's
arithmetic lives here.
"""
from .workloads import WORKLOADS, Workload, make_inputs, make_chain, prefix_inputs, head_params, as_float, group_of_head  # noqa: F401
