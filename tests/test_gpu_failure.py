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
