"""ctypes binding of libcrisp.so — argument marshalling only.

Every function here forwards to the C ABI declared in include/crisp.h. The
tensors are torch CUDA tensors (PyTorch provides device memory and streams);
all computation happens in the library's kernels. There is no fallback: if
the library cannot be loaded, importing it raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libcrisp.so")

CRISP_OK = 0
STATUS_NAMES = {0: "ok", -1: "invalid argument", -2: "unsupported shape", -3: "workspace too small",
                -4: "CUDA error", -5: "device wait timed out", -6: "device index out of range"}
ROUTER = {"cstruct": 0, "jsd": 1}
VS_RULE = {"alpha": 0, "gamma": 1, "alpha_median": 2}
GRANULARITY = {"tile": 0, "token": 1}
TILE_ID_MASK, TILE_WHOLE, TILE_SLASH_SHIFT = 0xFFFFFF, 1 << 24, 25
PATTERN_VS, PATTERN_PE = 0, 1

EXPORTED = ("crisp_version", "crisp_status_string", "crisp_check_params", "crisp_workspace_size",
            "crisp_route", "crisp_select", "crisp_sparse_prefill", "crisp_dense_prefill",
            "crisp_get_device_status", "crisp_route_noalloc", "crisp_selftest_wait_timeout",
            "crisp_selftest_pipeline_timeout", "crisp_prefill_host_workspace_size", "crisp_prefill_host")
NOALLOC_SCRATCH_BYTES = 16 << 20


class CrispError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({STATUS_NAMES.get(status, 'unknown')})")
        self.status = status


class CrispParams(ctypes.Structure):
    """Mirror of crisp_params (include/crisp.h)."""

    _fields_ = [("batch", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("seqlen", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("gamma", ctypes.c_float), ("tau_proxy", ctypes.c_float),
                ("tau_jsd", ctypes.c_float), ("k_min_blocks", ctypes.c_int32),
                ("router", ctypes.c_int32), ("vs_rule", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("vs_granularity", ctypes.c_int32), ("seq_lens", ctypes.c_void_p)]

    @property
    def n_blocks(self) -> int:
        """Blocks of the longest sequence (the stride of per-block outputs)."""
        return -(-self.seqlen // self.block)


def make_params(batch, h_q, h_kv, seqlen, head_dim, block=128, alpha=1.0, gamma=0.95,
                tau_proxy=0.2, tau_jsd=0.1, k_min_blocks=8, router="cstruct", vs_rule="alpha",
                sm_scale=0.0, seq_lens: Optional[torch.Tensor] = None, granularity="tile") -> CrispParams:
    """seq_lens: optional CUDA int32 tensor [batch] of sequence lengths. The
    params keep only its device address: keep the tensor alive while they are
    in use."""
    if seq_lens is not None:
        if not (seq_lens.is_cuda and seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
                and seq_lens.numel() == batch):
            raise ValueError("seq_lens must be a contiguous CUDA int32 tensor with one entry per batch element")
    p = CrispParams(batch, h_q, h_kv, seqlen, head_dim, block, alpha, gamma, tau_proxy, tau_jsd,
                    k_min_blocks, ROUTER[router] if isinstance(router, str) else int(router),
                    VS_RULE[vs_rule] if isinstance(vs_rule, str) else int(vs_rule), sm_scale,
                    GRANULARITY[granularity] if isinstance(granularity, str) else int(granularity),
                    None if seq_lens is None else seq_lens.data_ptr())
    return p


def params_for(q: torch.Tensor, k: torch.Tensor, **kw) -> CrispParams:
    b, hq, n, d = q.shape
    return make_params(b, hq, k.shape[1], n, d, **kw)


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libcrisp.so once and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libcrisp.so not built at {path}; run python -m dynamic_block_sparse_qk_b200.build")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(CrispParams)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    lib.crisp_version.restype = i32
    lib.crisp_status_string.restype = ctypes.c_char_p
    lib.crisp_status_string.argtypes = [i32]
    lib.crisp_check_params.restype = i32
    lib.crisp_check_params.argtypes = [P]
    lib.crisp_workspace_size.restype = sz
    lib.crisp_workspace_size.argtypes = [P]
    lib.crisp_route.restype = i32
    lib.crisp_route.argtypes = [P, vp, vp, vp, sz, vp, vp, vp, vp, vp]
    lib.crisp_select.restype = i32
    lib.crisp_select.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp, vp, vp]
    lib.crisp_sparse_prefill.restype = i32
    lib.crisp_sparse_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.crisp_dense_prefill.restype = i32
    lib.crisp_dense_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.crisp_route_noalloc.restype = i32
    lib.crisp_route_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
    lib.crisp_selftest_wait_timeout.restype = i32
    lib.crisp_selftest_wait_timeout.argtypes = [vp, ctypes.c_longlong, vp]
    lib.crisp_selftest_pipeline_timeout.restype = i32
    lib.crisp_selftest_pipeline_timeout.argtypes = [P, vp, vp, vp, vp, vp, sz, ctypes.c_longlong, vp]
    lib.crisp_prefill_host_workspace_size.restype = sz
    lib.crisp_prefill_host_workspace_size.argtypes = [P, i32]
    lib.crisp_prefill_host.restype = i32
    lib.crisp_prefill_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    lib.crisp_get_device_status.restype = i32
    lib.crisp_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), vp]
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, status: int):
    if status != CRISP_OK:
        raise CrispError(fn, status)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("CRISP tensors must live on a CUDA device")
        if t is not None and not t.is_contiguous():
            raise ValueError("CRISP tensors must be contiguous")


def crisp_workspace_size(p: CrispParams) -> int:
    n = load_library().crisp_workspace_size(ctypes.byref(p))
    if n == 0:
        _check("crisp_workspace_size", load_library().crisp_check_params(ctypes.byref(p)))
    return int(n)


def alloc_workspace(p: CrispParams, device="cuda") -> torch.Tensor:
    """Workspace tensor with its status word (first 8 bytes) cleared."""
    ws = torch.empty(crisp_workspace_size(p), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def crisp_route(p: CrispParams, q, k, ws, pattern=None, score=None, p_v=None, p_s=None, stream=None):
    """Algorithm 2 for every head. Returns (pattern, score, p_v, p_s)."""
    _need_cuda(q, k, ws)
    bh, nb = p.batch * p.h_q, p.n_blocks
    dev = q.device
    pattern = torch.empty(bh, dtype=torch.int32, device=dev) if pattern is None else pattern
    score = torch.empty(bh, dtype=torch.float32, device=dev) if score is None else score
    p_v = torch.empty(bh, nb, dtype=torch.float32, device=dev) if p_v is None else p_v
    p_s = torch.empty(bh, nb, dtype=torch.float32, device=dev) if p_s is None else p_s
    _check("crisp_route", load_library().crisp_route(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(ws), ws.numel(), _ptr(pattern), _ptr(score),
        _ptr(p_v), _ptr(p_s), _stream(stream)))
    return pattern, score, p_v, p_s


def crisp_select(p: CrispParams, q, k, pattern, p_v, p_s, ws, want_mask=True, mask=None,
                 tile_idx=None, tile_cnt=None, vs_sel=None, stream=None):
    """Algorithms 3/4/6 and tile lists. Returns (mask or None, tile_idx, tile_cnt).

    Pass a uint8 tensor [B*H_q, 2, N_b] as ``vs_sel`` to receive the selected
    vertical / slash block flags of VS heads."""
    _need_cuda(q, k, pattern, p_v, p_s, ws)
    bh, nb = p.batch * p.h_q, p.n_blocks
    dev = q.device
    if want_mask and mask is None:
        mask = torch.empty(bh, nb, nb, dtype=torch.uint8, device=dev)
    tile_idx = torch.empty(bh, nb, nb, dtype=torch.int32, device=dev) if tile_idx is None else tile_idx
    tile_cnt = torch.empty(bh, nb, dtype=torch.int32, device=dev) if tile_cnt is None else tile_cnt
    _check("crisp_select", load_library().crisp_select(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(pattern), _ptr(p_v), _ptr(p_s), _ptr(ws), ws.numel(),
        _ptr(mask), _ptr(vs_sel), _ptr(tile_idx), _ptr(tile_cnt), _stream(stream)))
    return mask, tile_idx, tile_cnt


def crisp_sparse_prefill(p: CrispParams, q, k, v, tile_idx, tile_cnt, ws, o=None, lse=None,
                         want_lse=True, stream=None):
    """Eq. 1 over the selected tiles. Returns (o, lse or None)."""
    _need_cuda(q, k, v, tile_idx, tile_cnt, ws)
    o = torch.empty_like(q) if o is None else o
    if want_lse and lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    _check("crisp_sparse_prefill", load_library().crisp_sparse_prefill(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(tile_idx), _ptr(tile_cnt), _ptr(o),
        _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse


def crisp_dense_prefill(p: CrispParams, q, k, v, ws, o=None, lse=None, want_lse=True, stream=None):
    """Dense causal attention with the same kernel. Returns (o, lse or None)."""
    _need_cuda(q, k, v, ws)
    o = torch.empty_like(q) if o is None else o
    if want_lse and lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    _check("crisp_dense_prefill", load_library().crisp_dense_prefill(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
        _stream(stream)))
    return o, lse


def crisp_route_noalloc(p: CrispParams, q, k, pattern=None, score=None, p_v=None, p_s=None,
                        stream=None):
    """Routing for callers that may not allocate device memory: the same
    kernels as crisp_route, with the library's fixed scratch array instead of
    a workspace. Returns (pattern, score, p_v, p_s). Output tensors passed in
    are used as given; when omitted they are created here by torch, which is
    this wrapper's convenience, not the library's."""
    _need_cuda(q, k)
    bh, nb = p.batch * p.h_q, p.n_blocks
    dev = q.device
    pattern = torch.empty(bh, dtype=torch.int32, device=dev) if pattern is None else pattern
    score = torch.empty(bh, dtype=torch.float32, device=dev) if score is None else score
    p_v = torch.empty(bh, nb, dtype=torch.float32, device=dev) if p_v is None else p_v
    p_s = torch.empty(bh, nb, dtype=torch.float32, device=dev) if p_s is None else p_s
    _check("crisp_route_noalloc", load_library().crisp_route_noalloc(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(pattern), _ptr(score), _ptr(p_v), _ptr(p_s),
        _stream(stream)))
    return pattern, score, p_v, p_s


def crisp_get_device_status(ws, stream=None) -> int:
    """Reads and clears the device status word of a workspace (ws = None:
    the scratch array of crisp_route_noalloc on the current device)."""
    st = ctypes.c_int32(0)
    _check("crisp_get_device_status",
           load_library().crisp_get_device_status(_ptr(ws), ctypes.byref(st), _stream(stream)))
    return int(st.value)


def crisp_prefill(q, k, v, ws=None, want_mask=False, stream=None, **kw):
    """Algorithm 1 end to end: route, select, sparse attention.

    Returns a dict with o, lse, pattern, score, p_v, p_s, tile_idx, tile_cnt
    (and mask when requested)."""
    p = params_for(q, k, **kw)
    ws = alloc_workspace(p, q.device) if ws is None else ws
    pattern, score, p_v, p_s = crisp_route(p, q, k, ws, stream=stream)
    mask, tile_idx, tile_cnt = crisp_select(p, q, k, pattern, p_v, p_s, ws, want_mask=want_mask,
                                            stream=stream)
    o, lse = crisp_sparse_prefill(p, q, k, v, tile_idx, tile_cnt, ws, stream=stream)
    return {"o": o, "lse": lse, "pattern": pattern, "score": score, "p_v": p_v, "p_s": p_s,
            "mask": mask, "tile_idx": tile_idx, "tile_cnt": tile_cnt, "params": p, "ws": ws}


def crisp_selftest_wait_timeout(ws: torch.Tensor, limit_cycles: int = 1 << 20, stream=None) -> None:
    """Runs the bounded-wait self-test on ws's device (see include/crisp.h):
    afterwards crisp_get_device_status(ws) reports CRISP_ERR_TIMEOUT (-5)."""
    _need_cuda(ws)
    _check("crisp_selftest_wait_timeout", load_library().crisp_selftest_wait_timeout(
        _ptr(ws), int(limit_cycles), _stream(stream)))


def crisp_selftest_pipeline_timeout(p: CrispParams, q, k, v, o, ws, limit_cycles: int = 64,
                                    stream=None) -> None:
    """Runs the proxy and attention kernels with every pipeline wait cut to
    ``limit_cycles`` (see include/crisp.h): afterwards
    crisp_get_device_status(ws) reports CRISP_ERR_TIMEOUT (-5)."""
    _need_cuda(q, k, v, o, ws)
    _check("crisp_selftest_pipeline_timeout", load_library().crisp_selftest_pipeline_timeout(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ws), ws.numel(), int(limit_cycles),
        _stream(stream)))


def crisp_prefill_host_workspace_size(p: CrispParams, kv_per_chunk: int = 1) -> int:
    n = load_library().crisp_prefill_host_workspace_size(ctypes.byref(p), int(kv_per_chunk))
    if n == 0:
        _check("crisp_prefill_host_workspace_size", load_library().crisp_check_params(ctypes.byref(p)))
        raise CrispError("crisp_prefill_host_workspace_size", -1)
    return int(n)


def crisp_prefill_host(p: CrispParams, q, k, v, o, ws, lse=None, seq_lens=None, pattern=None,
                       kv_per_chunk: int = 1, stream=None) -> None:
    """The whole prefill on pinned host tensors (see include/crisp.h):
    synchronous; ``seq_lens`` a host int32 tensor or None, ``pattern`` an
    optional host int32 tensor [batch * h_q] receiving the routes, ``ws`` a
    device uint8 tensor of crisp_prefill_host_workspace_size bytes."""
    _need_cuda(ws)
    for t in (q, k, v, o, lse, seq_lens, pattern):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("crisp_prefill_host takes contiguous host tensors")
    n, d = p.seqlen, p.head_dim
    want = {"q": (q, (p.batch, p.h_q, n, d), torch.bfloat16), "k": (k, (p.batch, p.h_kv, n, d), torch.bfloat16),
            "v": (v, (p.batch, p.h_kv, n, d), torch.bfloat16), "o": (o, (p.batch, p.h_q, n, d), torch.bfloat16),
            "lse": (lse, (p.batch, p.h_q, n), torch.float32), "seq_lens": (seq_lens, (p.batch,), torch.int32),
            "pattern": (pattern, (p.batch * p.h_q,), torch.int32)}
    for name, (t, shape, dtype) in want.items():
        if t is not None and (t.dtype != dtype or t.numel() != math.prod(shape)):
            raise ValueError(f"{name} must hold {math.prod(shape)} elements of {dtype}")
    _check("crisp_prefill_host", load_library().crisp_prefill_host(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(seq_lens), _ptr(pattern),
        int(kv_per_chunk), _ptr(ws), ws.numel(), _stream(stream)))
