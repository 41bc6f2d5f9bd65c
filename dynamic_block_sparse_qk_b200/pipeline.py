"""CRISP prefill of host-resident inputs, pipelined over KV-head groups.

Every query head with its KV head is an independent problem (GQA groups
share nothing across KV heads), so a prefill whose Q, K, V live in (pinned)
host memory can be cut into chunks of KV heads: while the kernels of chunk i
run, the inputs of chunk i+1 travel host-to-device and the output of chunk
i-1 travels device-to-host. Three CUDA streams carry the copies in, the
compute and the copies out; two slots of device buffers alternate between
chunks. Every compute step is a call through the C ABI (crisp_route,
crisp_select, crisp_sparse_prefill); this module only moves memory and
orders streams.

With per-sequence lengths only the rows a sequence holds cross PCIe (one
copy per head); rows of o (and lse) past a sequence's length are left as
they were on the host.

The call is asynchronous with respect to the host and ordered on the
caller's current stream: the pipeline starts after the work already queued
there and the current stream waits for its last copy.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


def _pinned(t: torch.Tensor, name: str):
    if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor in pinned host memory")


def prefill_from_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                      lse: Optional[torch.Tensor] = None, seq_lens: Optional[list] = None,
                      kv_per_chunk: int = 1, device=None, **params) -> dict:
    """Sparse prefill of host tensors q [B, H_q, N, d], k, v [B, H_kv, N, d]
    (bf16, pinned) into the pinned host tensor o (and lse [B, H_q, N] fp32 if
    given). ``seq_lens``: optional per-batch lengths (host ints). ``params``:
    the hyper-parameters of make_params (block, alpha, gamma, router, ...).

    Returns a dict of per-chunk device outputs kept for inspection:
    {"pattern": [B*H_q] int32 on the device, "tile_cnt_sum": device scalar}.
    """
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _pinned(t, nm)
    if lse is not None:
        _pinned(lse, "lse")
    bsz, hq, n, d = q.shape
    hkv = k.shape[1]
    if hkv % kv_per_chunk:
        raise ValueError("kv_per_chunk must divide the number of KV heads")
    g = hq // hkv
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    caller = torch.cuda.current_stream(dev)
    ck, cq = kv_per_chunk, kv_per_chunk * g
    lens_dev = [None] * bsz
    if seq_lens is not None:
        for b in range(bsz):
            lens_dev[b] = torch.tensor([int(seq_lens[b])], dtype=torch.int32, device=dev)
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    start = torch.cuda.Event()
    start.record(caller)
    for s in (s_in, s_cmp, s_out):
        s.wait_event(start)
    p = B.make_params(1, cq, ck, n, d, **params)
    nb = p.n_blocks
    with torch.cuda.stream(s_cmp):
        slots = []
        for _ in range(2):
            ws = torch.empty(B.crisp_workspace_size(p), dtype=torch.uint8, device=dev)
            ws[:256].zero_()
            slots.append({
                # rows past a sequence keep older (finite) contents; v starts at
                # zero because those rows of its last tile meet exact-zero weights
                "q": torch.empty((1, cq, n, d), dtype=q.dtype, device=dev),
                "k": torch.empty((1, ck, n, d), dtype=k.dtype, device=dev),
                "v": torch.zeros((1, ck, n, d), dtype=v.dtype, device=dev),
                "o": torch.empty((1, cq, n, d), dtype=q.dtype, device=dev),
                "lse": torch.empty((1, cq, n), dtype=torch.float32, device=dev) if lse is not None else None,
                "ws": ws,
                "pattern": torch.empty(cq, dtype=torch.int32, device=dev),
                "score": torch.empty(cq, dtype=torch.float32, device=dev),
                "p_v": torch.empty(cq, nb, dtype=torch.float32, device=dev),
                "p_s": torch.empty(cq, nb, dtype=torch.float32, device=dev),
                "tidx": torch.empty(cq, nb, nb, dtype=torch.int32, device=dev),
                "tcnt": torch.empty(cq, nb, dtype=torch.int32, device=dev),
                "in": torch.cuda.Event(), "cmp": torch.cuda.Event(), "out": torch.cuda.Event(),
                "used": False,
            })
    with torch.cuda.stream(s_cmp):
        pattern_all = torch.empty(bsz * hq, dtype=torch.int32, device=dev)
        tiles = torch.zeros((), dtype=torch.int64, device=dev)
    chunks = [(b, h0) for b in range(bsz) for h0 in range(0, hkv, ck)]
    for ci, (b, h0) in enumerate(chunks):
        sl = slots[ci % 2]
        qs = slice(h0 * g, h0 * g + cq)
        ks = slice(h0, h0 + ck)
        # inputs of this slot are free once the compute of its previous chunk ended
        if sl["used"]:
            s_in.wait_event(sl["cmp"])
        nv = n if seq_lens is None else int(seq_lens[b])
        with torch.cuda.stream(s_in):
            if nv == n:
                sl["q"][0].copy_(q[b, qs], non_blocking=True)
                sl["k"][0].copy_(k[b, ks], non_blocking=True)
                sl["v"][0].copy_(v[b, ks], non_blocking=True)
            else:                                            # the sequence's rows only, per head
                for hh in range(cq):
                    sl["q"][0, hh, :nv].copy_(q[b, qs.start + hh, :nv], non_blocking=True)
                for hh in range(ck):
                    sl["k"][0, hh, :nv].copy_(k[b, ks.start + hh, :nv], non_blocking=True)
                    sl["v"][0, hh, :nv].copy_(v[b, ks.start + hh, :nv], non_blocking=True)
        sl["in"].record(s_in)
        # outputs of this slot are free once its previous copy out ended
        s_cmp.wait_event(sl["in"])
        if sl["used"]:
            s_cmp.wait_event(sl["out"])
        pc = B.make_params(1, cq, ck, n, d, seq_lens=lens_dev[b], **params)
        B.crisp_route(pc, sl["q"], sl["k"], sl["ws"], sl["pattern"], sl["score"], sl["p_v"], sl["p_s"],
                      stream=s_cmp)
        B.crisp_select(pc, sl["q"], sl["k"], sl["pattern"], sl["p_v"], sl["p_s"], sl["ws"], want_mask=False,
                       tile_idx=sl["tidx"], tile_cnt=sl["tcnt"], stream=s_cmp)
        B.crisp_sparse_prefill(pc, sl["q"], sl["k"], sl["v"], sl["tidx"], sl["tcnt"], sl["ws"], o=sl["o"],
                               lse=sl["lse"], want_lse=lse is not None, stream=s_cmp)
        with torch.cuda.stream(s_cmp):
            pattern_all[b * hq + h0 * g: b * hq + h0 * g + cq].copy_(sl["pattern"])
            tiles.add_(sl["tcnt"].sum())
        sl["cmp"].record(s_cmp)
        s_out.wait_event(sl["cmp"])
        with torch.cuda.stream(s_out):
            if nv == n:
                o[b, qs].copy_(sl["o"][0], non_blocking=True)
                if lse is not None:
                    lse[b, qs].copy_(sl["lse"][0], non_blocking=True)
            else:
                for hh in range(cq):
                    o[b, qs.start + hh, :nv].copy_(sl["o"][0, hh, :nv], non_blocking=True)
                    if lse is not None:
                        lse[b, qs.start + hh, :nv].copy_(sl["lse"][0, hh, :nv], non_blocking=True)
        sl["out"].record(s_out)
        sl["used"] = True
    # the caller's stream continues after the last copy out and the last compute
    for s in (s_in, s_cmp, s_out):
        done = torch.cuda.Event()
        done.record(s)
        caller.wait_event(done)
    # device buffers may be reused by the allocator only after the streams that
    # touched them are done
    for sl in slots:
        for key, val in sl.items():
            if isinstance(val, torch.Tensor):
                for s in (s_in, s_cmp, s_out):
                    val.record_stream(s)
    for t in list(lens_dev) + [pattern_all, tiles]:
        if t is not None:
            t.record_stream(s_cmp)
    return {"pattern": pattern_all, "tile_cnt_sum": tiles}
