"""crisp_route_noalloc: routing for callers that may not allocate device memory.

Such callers (a plug-in whose host framework keeps all device memory in its
own pool and passes no workspace, or a serving loop that cannot take the
synchronisation cudaMalloc may cause) get the same routing kernels with a
fixed scratch array compiled into the library. These tests call the new entry
point through the C ABI and check it against crisp_route, which uses a
caller workspace: equal patterns, scores and block scores (within the
tolerance of the other parity tests) on consecutive calls that share the
array, a clean rejection of problems too large for it, and that a device-side
error of a call lands in the array's status word, which
crisp_get_device_status(NULL) reads and clears.
"""
import ctypes

import pytest
import torch

from synthetic import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu

RTOL = 2e-5


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_block_sparse_qk_b200 import build, binding
    build.build()
    return binding


def _via_workspace(B, p, q, k):
    ws = B.alloc_workspace(p, q.device)
    out = B.crisp_route(p, q, k, ws)
    torch.cuda.synchronize()
    return out


def _via_noalloc_cabi(B, p, q, k):
    """Direct C-ABI call with caller-owned outputs (nothing allocated inside)."""
    lib = B.load_library()
    bh, nb = p.batch * p.h_q, p.n_blocks
    pattern = torch.full((bh,), -7, dtype=torch.int32, device=q.device)
    score = torch.full((bh,), float("nan"), dtype=torch.float32, device=q.device)
    p_v = torch.full((bh, nb), float("nan"), dtype=torch.float32, device=q.device)
    p_s = torch.full((bh, nb), float("nan"), dtype=torch.float32, device=q.device)
    st = lib.crisp_route_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                 ctypes.c_void_p(pattern.data_ptr()), ctypes.c_void_p(score.data_ptr()),
                                 ctypes.c_void_p(p_v.data_ptr()), ctypes.c_void_p(p_s.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st
    torch.cuda.synchronize()
    return pattern, score, p_v, p_s


def _same(a, b):
    assert torch.equal(a[0], b[0])
    for x, y in zip(a[1:], b[1:]):
        torch.testing.assert_close(x, y, rtol=RTOL, atol=1e-9)


def _problem(w, **kw):
    from dynamic_block_sparse_qk_b200 import binding as B
    q, k, _, _ = make_qkv(w)
    q, k = q.cuda(), k.cuda()
    return B.params_for(q, k, block=w.block, **kw), q, k


def test_matches_workspace_route_on_consecutive_calls(lib):
    # two different problems, then the first again: the shared array keeps the
    # previous call's contents, which must not leak into the next result
    cases = [_problem(WORKLOADS["tiny"]),
             _problem(Workload("mid", 1, 8, 2, 128, 8192, 128), router="jsd"),
             _problem(WORKLOADS["tiny"])]
    for p, q, k in cases:
        ref = _via_workspace(lib, p, q, k)
        first = _via_noalloc_cabi(lib, p, q, k)
        second = _via_noalloc_cabi(lib, p, q, k)
        _same(first, ref)
        _same(second, ref)


def test_largest_supported_problem_and_rejection(lib):
    p, q, k = _problem(WORKLOADS["llama_32k"])
    _same(_via_noalloc_cabi(lib, p, q, k), _via_workspace(lib, p, q, k))
    big = lib.make_params(1, 32, 8, 65536, 128, block=128)
    z = ctypes.c_void_p(1 << 20)
    assert lib.load_library().crisp_route_noalloc(ctypes.byref(big), z, z, z, z, z, z, None) == -3


def test_device_errors_reach_the_status_reader(lib):
    # a sequence length below 2 * block + 1 is clamped by the kernels and
    # reported as CRISP_ERR_DEVICE in the array's status word; the reader with
    # a NULL workspace returns it once and clears it
    w = WORKLOADS["tiny"]
    q, k, _, _ = make_qkv(w)
    q, k = q.cuda(), k.cuda()
    assert lib.crisp_get_device_status(None) == 0                 # whatever an earlier call left
    lens = torch.tensor([2 * w.block], dtype=torch.int32, device="cuda")
    p = lib.params_for(q, k, block=w.block, seq_lens=lens)
    _via_noalloc_cabi(lib, p, q, k)
    assert lib.crisp_get_device_status(None) == -6                # CRISP_ERR_DEVICE
    assert lib.crisp_get_device_status(None) == 0
    ok = lib.params_for(q, k, block=w.block)
    _same(_via_noalloc_cabi(lib, ok, q, k), _via_workspace(lib, ok, q, k))
    assert lib.crisp_get_device_status(None) == 0
