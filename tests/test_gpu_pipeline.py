"""Host-input prefill pipelined over KV-head groups (dynamic_block_sparse_qk_b200.pipeline):
the same results as the device-resident path, per head, with the copies of
one group overlapping the kernels of the next."""
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
    torch.cuda.synchronize()
    assert torch.equal(out["pattern"].cpu(), pattern.cpu())
    assert int(out["tile_cnt_sum"]) == int(tcnt.sum())
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
