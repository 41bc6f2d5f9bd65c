"""Host-input prefill through the C ABI's crisp_prefill_host (pipelined over
KV-head groups): the same results as the device-resident path, per head,
with the copies of one group overlapping the kernels of the next."""
import pytest
import torch

from synthetic import Workload, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_block_sparse_qk_b200 import build
    build.build()


@pytest.mark.parametrize("kv_per_chunk", [1, 2])
def test_pipeline_matches_device_path(kv_per_chunk):
    import dynamic_block_sparse_qk_b200 as C
    w = Workload("pipe", 2, 8, 4, 128, 4096 + 77, 128, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0,
                 lengths=(4096 + 77, 3000))
    q, k, v, _ = make_qkv(w)
    # device-resident reference: one call per stage over the whole batch
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lens = torch.tensor(w.lengths, dtype=torch.int32, device="cuda")
    p = C.params_for(qd, kd, block=128, seq_lens=lens)
    ws = C.alloc_workspace(p)
    pattern, score, p_v, p_s = C.crisp_route(p, qd, kd, ws)
    _, tidx, tcnt = C.crisp_select(p, qd, kd, pattern, p_v, p_s, ws, want_mask=False)
    o_ref, lse_ref = C.crisp_sparse_prefill(p, qd, kd, vd, tidx, tcnt, ws)
    assert C.crisp_get_device_status(ws) == 0
    # pinned host inputs through the pipeline
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    ho = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hl = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
    out = C.prefill_from_host(hq, hk, hv, ho, lse=hl, seq_lens=list(w.lengths), kv_per_chunk=kv_per_chunk,
                              block=128)
    assert torch.equal(out["pattern"], pattern.cpu())
    o_ref, lse_ref = o_ref.cpu(), lse_ref.cpu()
    for b, n in enumerate(w.lengths):                  # only a sequence's own rows are copied back
        err = (ho[b, :, :n].float() - o_ref[b, :, :n].float()).abs()
        assert float(err.max()) <= 2e-2 and float(err.mean()) <= 2e-3
        assert torch.allclose(hl[b, :, :n], lse_ref[b, :, :n], atol=2e-3, rtol=0)


def test_pipeline_rejects_pageable_inputs():
    import dynamic_block_sparse_qk_b200 as C
    x = torch.zeros(1, 2, 512, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        C.prefill_from_host(x, x[:, :1], x[:, :1], x.clone(), block=64)


def test_host_prefill_c_abi_direct_and_errors():
    # the entry point called straight through ctypes with pinned buffers:
    # the same output as the device path, a pageable buffer refused before
    # any copy, and a length out of range refused as a shape error
    import ctypes
    import dynamic_block_sparse_qk_b200 as C
    from dynamic_block_sparse_qk_b200 import binding as B
    w = Workload("pipe2", 1, 4, 2, 64, 2048, 64, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    q, k, v, _ = make_qkv(w)
    ref = C.crisp_prefill(q.cuda(), k.cuda(), v.cuda(), block=64)
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    ho = torch.zeros(q.shape, dtype=q.dtype).pin_memory()
    p = B.make_params(1, 4, 2, 2048, 64, block=64)
    ws = torch.empty(B.crisp_prefill_host_workspace_size(p, 2), dtype=torch.uint8, device="cuda")
    pat = torch.empty(4, dtype=torch.int32)
    lib = B.load_library()
    vp = ctypes.c_void_p
    st = lib.crisp_prefill_host(ctypes.byref(p), vp(hq.data_ptr()), vp(hk.data_ptr()), vp(hv.data_ptr()),
                                vp(ho.data_ptr()), None, None, vp(pat.data_ptr()), 2, vp(ws.data_ptr()),
                                ws.numel(), vp(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert torch.equal(pat, ref["pattern"].cpu())
    err = (ho.float() - ref["o"].cpu().float()).abs()
    assert float(err.max()) <= 2e-2 and float(err.mean()) <= 2e-3
    pageable = q.clone()
    assert lib.crisp_prefill_host(ctypes.byref(p), vp(pageable.data_ptr()), vp(hk.data_ptr()), vp(hv.data_ptr()),
                                  vp(ho.data_ptr()), None, None, None, 2, vp(ws.data_ptr()), ws.numel(),
                                  None) == -1
    bad = torch.tensor([100], dtype=torch.int32)             # <= 2 * block
    assert lib.crisp_prefill_host(ctypes.byref(p), vp(hq.data_ptr()), vp(hk.data_ptr()), vp(hv.data_ptr()),
                                  vp(ho.data_ptr()), None, vp(bad.data_ptr()), None, 2, vp(ws.data_ptr()),
                                  ws.numel(), None) == -2
