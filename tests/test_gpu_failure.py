"""Failure detection without a GPU fault: the bounded wait that every
pipelined kernel uses gives up after its cycle limit, records
CRISP_ERR_TIMEOUT in the workspace status word and returns; the context
stays usable for the next prefill."""
import pytest
import torch

from synthetic import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_block_sparse_qk_b200 import build
    build.build()


def test_bounded_wait_reports_timeout_and_context_survives():
    import dynamic_block_sparse_qk_b200 as C
    from dynamic_block_sparse_qk_b200 import binding as B
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    B.crisp_selftest_wait_timeout(ws, limit_cycles=1 << 20)        # well under a millisecond
    assert C.crisp_get_device_status(ws) == -5                       # CRISP_ERR_TIMEOUT
    assert C.crisp_get_device_status(ws) == 0                        # reading clears it
    # the next prefill on the same device runs normally
    q, k, v, _ = make_qkv(WORKLOADS["tiny"])
    out = C.crisp_prefill(q.cuda(), k.cuda(), v.cuda(), block=64)
    assert C.crisp_get_device_status(out["ws"]) == 0
    assert torch.isfinite(out["o"].float()).all()


@pytest.mark.parametrize("kw", [
    dict(seqlen=2048, block=128, head_dim=128, h_q=4, h_kv=2),
    dict(seqlen=2048 + 37, block=64, head_dim=64, h_q=2, h_kv=1),
    dict(seqlen=1024, block=64, head_dim=128, h_q=2, h_kv=2),
])
def test_pipelined_kernels_abort_cleanly_and_next_prefill_is_exact(kw):
    # The proxy and attention kernels run with every pipeline wait cut to 64
    # cycles, so their waits run out: each CTA records CRISP_ERR_TIMEOUT,
    # drains its copies and tensor-core operations and frees its tensor
    # memory. The context stays usable and the next prefill on the same
    # workspace matches the oracle.
    import numpy as np
    import oracle as O
    import dynamic_block_sparse_qk_b200 as C
    from dynamic_block_sparse_qk_b200 import binding as B
    from synthetic import Workload
    import parity_util as PU
    base = dict(name="abort", batch=1, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    base.update(kw)
    w = Workload(**base)
    q, k, v, _ = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = C.params_for(qd, kd, block=w.block)
    ws = C.alloc_workspace(p)
    o = torch.empty_like(qd)
    B.crisp_selftest_pipeline_timeout(p, qd, kd, vd, o, ws, limit_cycles=64)
    assert C.crisp_get_device_status(ws) == -5                       # CRISP_ERR_TIMEOUT
    assert C.crisp_get_device_status(ws) == 0
    gpu = PU.run_gpu(w, q, k, v)
    assert gpu["status"] == 0
    PU.compare_all(w, q, k, v, gpu, PU.oracle_params(w))
    od, _ = C.crisp_dense_prefill(p, qd, kd, vd, ws)
    assert C.crisp_get_device_status(ws) == 0
    nb = O.n_blocks(w.seqlen, w.block)
    full = np.tril(np.ones((nb, nb), dtype=bool))
    g = w.h_q // w.h_kv
    for h in range(w.h_q):
        ref, _, rows = O.masked_attention_rows(O.bf16_to_f64(q[0, h]), O.bf16_to_f64(k[0, h // g]),
                                               O.bf16_to_f64(v[0, h // g]), full, w.block, w.head_dim ** -0.5)
        err = np.abs(od[0, h].float().cpu().numpy()[rows] - ref)
        assert err.max() <= PU.ATTN_MAX_ABS and err.mean() <= PU.ATTN_MEAN_ABS
