"""B200-native CRISP sparse attention prefill (sm_100a kernels behind a C ABI).

Stages (CRISP paper, Algorithm 1): crisp_route (PatSearch, Algorithm 2),
crisp_select (Algorithms 3, 4 and 6 plus tile lists), crisp_sparse_prefill
(block-sparse attention, Eq. 1) and crisp_dense_prefill (the same kernel
over every causal tile); prefill_from_host calls the library's
crisp_prefill_host, which runs the three stages on pinned host inputs,
overlapping the PCIe copies of one KV-head group with the kernels of the
next.
"""
from .binding import (CrispError, CrispParams, PATTERN_PE, PATTERN_VS, alloc_workspace,
                      crisp_dense_prefill, crisp_get_device_status, crisp_prefill, crisp_route,
                      crisp_select, crisp_sparse_prefill, crisp_workspace_size, load_library,
                      make_params, params_for)
from .pipeline import host_workspace, prefill_from_host

__all__ = ["CrispError", "CrispParams", "PATTERN_PE", "PATTERN_VS", "alloc_workspace",
           "crisp_dense_prefill", "crisp_get_device_status", "crisp_prefill", "crisp_route",
           "crisp_select", "crisp_sparse_prefill", "crisp_workspace_size", "load_library",
           "make_params", "params_for", "host_workspace", "prefill_from_host"]
