"""CRISP prefill of host-resident inputs: a thin caller of the C ABI's
crisp_prefill_host.

Every query head with its KV head is an independent problem (GQA groups
share nothing across KV heads), so the library cuts a prefill whose Q, K, V
live in pinned host memory into chunks of KV heads: while the kernels of
chunk i run, the inputs of chunk i+1 travel host-to-device and the output of
chunk i-1 travels device-to-host (two slots of device buffers in the
caller's workspace, the copies on two streams of their own). This module
only checks the tensors, sizes the workspace and marshals the call.

With per-sequence lengths only the rows a sequence holds cross PCIe; rows
of o (and lse) past a sequence's length are left as they were on the host.
The call is synchronous and raises CrispError on any error, kernel-side
errors (a wait that ran out, an out-of-range index) included.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


def _pinned(t: torch.Tensor, name: str):
    if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor in pinned host memory")


def host_workspace(q: torch.Tensor, k: torch.Tensor, kv_per_chunk: int = 1, device=None,
                   **params) -> torch.Tensor:
    """Device workspace for prefill_from_host on tensors shaped like q, k."""
    bsz, hq, n, d = q.shape
    p = B.make_params(bsz, hq, k.shape[1], n, d, **params)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.empty(B.crisp_prefill_host_workspace_size(p, kv_per_chunk), dtype=torch.uint8, device=dev)


def prefill_from_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                      lse: Optional[torch.Tensor] = None, seq_lens: Optional[list] = None,
                      kv_per_chunk: int = 1, device=None, ws: Optional[torch.Tensor] = None,
                      **params) -> dict:
    """Sparse prefill of host tensors q [B, H_q, N, d], k, v [B, H_kv, N, d]
    (bf16, pinned) into the pinned host tensor o (and lse [B, H_q, N] fp32 if
    given). ``seq_lens``: optional per-batch lengths (host ints). ``ws``: an
    optional device workspace from host_workspace (created here otherwise).
    ``params``: the hyper-parameters of make_params (block, alpha, gamma,
    router, ...).

    Returns {"pattern": host int32 tensor [B*H_q]} (the route of every head).
    """
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _pinned(t, nm)
    if lse is not None:
        _pinned(lse, "lse")
    bsz, hq, n, d = q.shape
    p = B.make_params(bsz, hq, k.shape[1], n, d, **params)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if ws is None:
        ws = torch.empty(B.crisp_prefill_host_workspace_size(p, kv_per_chunk), dtype=torch.uint8, device=dev)
    lens = None if seq_lens is None else torch.tensor([int(x) for x in seq_lens], dtype=torch.int32)
    pattern = torch.empty(bsz * hq, dtype=torch.int32)
    with torch.cuda.device(dev):
        B.crisp_prefill_host(p, q, k, v, o, ws, lse=lse, seq_lens=lens, pattern=pattern,
                             kv_per_chunk=kv_per_chunk, stream=torch.cuda.current_stream(dev))
    return {"pattern": pattern}
