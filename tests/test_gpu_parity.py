"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Routing and selected blocks are compared exactly outside the 1e-4 exemption
band; attention against the oracle run on the GPU's own mask (max-abs 2e-2,
mean-abs 2e-3). Larger configs sample query blocks for attention and check
routing and selection in full.
"""
import numpy as np
import pytest
import torch

import oracle as O
from synthetic import WORKLOADS, Workload, make_qkv, sweep_workload
import parity_util as PU

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_block_sparse_qk_b200 import build
    build.build()


def _check(w, router="cstruct", vs_rule="alpha", alpha=1.0, gamma=0.95, qblocks_fn=None,
           heads=None, expect_both=False, granularity="tile", inputs=None, keep_on_device=False):
    q, k, v, meta = make_qkv(w) if inputs is None else inputs
    gpu = PU.run_gpu(w, q, k, v, router=router, vs_rule=vs_rule, alpha=alpha, gamma=gamma,
                     granularity=granularity, keep_on_device=keep_on_device)
    assert gpu["status"] == 0
    oprm = PU.oracle_params(w, router=router, vs_rule=vs_rule, alpha=alpha, gamma=gamma,
                            granularity=granularity)
    reps = PU.compare_all(w, q, k, v, gpu, oprm, qblocks_fn=qblocks_fn, heads=heads)
    PU.record(f"{w.name} {router} {vs_rule} alpha={alpha} gamma={gamma} {granularity}", reps)
    if expect_both:
        pats = {r["pattern"] for r in reps}
        assert pats == {O.VS, O.PE}, pats
    return reps


def _device_inputs(w):
    """Inputs generated on the GPU (fast at 64k-512k), copied to the host for
    the oracle; the CUDA path receives the same values."""
    q, k, v, meta = make_qkv(w, device="cuda")
    out = (q.cpu(), k.cpu(), v.cpu(), meta)
    del q, k, v
    torch.cuda.empty_cache()
    return out


def _check_alphas(w, alphas, qblocks_fn, inputs, expect_both=False, vs_rules=None):
    """One input, several alpha values (or VS rules): each is a full GPU
    prefill (route, select, attention) compared with the oracle; the oracle
    routes and runs the PE index once per head and the VS index once per
    setting."""
    q, k, v, _ = inputs
    vs_rules = vs_rules or ["alpha"] * len(alphas)
    oprms = [PU.oracle_params(w, alpha=a, vs_rule=r) for a, r in zip(alphas, vs_rules)]
    gpus = []
    for a, r in zip(alphas, vs_rules):
        gpu = PU.run_gpu(w, q, k, v, alpha=a, vs_rule=r, keep_on_device=True)
        assert gpu["status"] == 0
        gpus.append(gpu)
    g = w.h_q // w.h_kv
    reps = [[] for _ in alphas]
    kv_cache = {}
    for h in range(w.h_q):
        if h // g not in kv_cache:
            kv_cache = {h // g: (O.bf16_to_f64(k[0, h // g]), O.bf16_to_f64(v[0, h // g]))}
        kh, vh = kv_cache[h // g]
        qh = O.bf16_to_f64(q[0, h])
        orcs = PU.oracle_for_alphas(qh, kh, oprms)
        for i in range(len(alphas)):
            reps[i].append(PU.compare_head(gpus[i], 0, h, qh, kh, vh, w, oprms[i], qblocks_fn(i, h),
                                           orc=orcs[i]))
    for i, a in enumerate(alphas):
        PU.record(f"{w.name} cstruct {vs_rules[i]} alpha={a} gamma=0.95 tile", reps[i])
        if expect_both:
            assert {r["pattern"] for r in reps[i]} == {O.VS, O.PE}
    return reps


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.0])
def test_tiny_full(alpha):
    reps = _check(WORKLOADS["tiny"], alpha=alpha, expect_both=True)
    assert reps[0]["pattern"] == O.VS and reps[1]["pattern"] == O.PE


def test_tiny_gamma_vs_rule():          # Abl.1: C_struct routing + gamma VS selection
    _check(WORKLOADS["tiny"], vs_rule="gamma")


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.0])
def test_tiny_median_floor(alpha):      # Appendix H: median noise floor in the alpha rule
    _check(WORKLOADS["tiny"], vs_rule="alpha_median", alpha=alpha, expect_both=True)


@pytest.mark.parametrize("kw", [
    dict(seqlen=384, block=128, head_dim=128, h_q=2, h_kv=1),              # N_b = 3: one middle block
    dict(seqlen=768, block=128, head_dim=64, h_q=4, h_kv=2),               # N_b = 6: even middle count
    dict(seqlen=1024, block=64, head_dim=128, h_q=3, h_kv=3),              # N_b = 16, B = 64
])
def test_edge_shapes_median_floor(kw):
    base = dict(name="edge", batch=1, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    base.update(kw)
    _check(Workload(**base), vs_rule="alpha_median")


def test_tiny_jsd_router():             # Abl.2: JSD routing + alpha VS selection
    _check(WORKLOADS["tiny"], router="jsd")


def test_tiny_unit_variance_values():   # V ~ N(0,1): the absolute tolerance bites
    reps = _check(WORKLOADS["tiny"].with_(v_unit=True))
    assert max(r["attn_max_abs"] for r in reps) < 2e-2


@pytest.mark.parametrize("kw", [
    dict(seqlen=384, block=128, head_dim=128, h_q=2, h_kv=1),              # N_b = 3 (smallest)
    dict(seqlen=640, block=128, head_dim=64, h_q=4, h_kv=2),               # odd N_b, d=64 at B=128
    dict(seqlen=1024, block=64, head_dim=128, h_q=3, h_kv=3),              # B=64 with d=128, g=1
    dict(seqlen=1536, block=128, head_dim=128, h_q=4, h_kv=1, batch=2),    # batch 2, GQA g=4
])
def test_edge_shapes(kw):
    base = dict(name="edge", batch=1, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    base.update(kw)
    _check(Workload(**base))


# ---- sequences whose length is not a multiple of the block (N_b = ceil(n / B)),
# and batches of different lengths stored with padding rows
@pytest.mark.parametrize("kw", [
    dict(seqlen=2048 + 37, block=64, head_dim=64, h_q=2, h_kv=1),          # tiny shape, 37-row last block
    dict(seqlen=5 * 128 + 1, block=128, head_dim=128, h_q=4, h_kv=2),      # one-token last block
    dict(seqlen=3 * 128 - 1, block=128, head_dim=128, h_q=2, h_kv=1),      # N_b = 3, 127-row last block
    dict(seqlen=1000, block=64, head_dim=64, h_q=4, h_kv=1),               # GQA g = 4, 40-row last block
    dict(seqlen=4096 + 77, block=128, head_dim=64, h_q=2, h_kv=2),         # d = 64 at B = 128
])
def test_ragged_single_sequence(kw):
    base = dict(name="ragged", batch=1, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    base.update(kw)
    _check(Workload(**base))


@pytest.mark.parametrize("router,vs_rule", [("jsd", "alpha"), ("cstruct", "gamma"), ("cstruct", "alpha_median")])
def test_ragged_router_and_rules(router, vs_rule):
    w = Workload("ragged_r", 1, 4, 2, 128, 2048 + 93, 128, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    _check(w, router=router, vs_rule=vs_rule)


@pytest.mark.parametrize("kw", [
    dict(batch=3, seqlen=2048, block=128, head_dim=128, h_q=4, h_kv=2, lengths=(2048, 1500, 257)),
    dict(batch=2, seqlen=1536 + 64, block=64, head_dim=64, h_q=2, h_kv=1, lengths=(777, 1600)),
    dict(batch=2, seqlen=4096, block=128, head_dim=128, h_q=8, h_kv=2, lengths=(4096 - 1, 2 * 128 + 1)),
])
def test_variable_length_batch(kw):
    base = dict(name="varlen", n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    base.update(kw)
    _check(Workload(**base))


@pytest.mark.parametrize("router,vs_rule", [("jsd", "gamma"), ("cstruct", "alpha_median")])
def test_variable_length_batch_routers_and_rules(router, vs_rule):
    w = Workload("varlen_r", 3, 4, 2, 128, 2048 + 64, 128, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0,
                 lengths=(2048 + 64, 1111, 3 * 128 + 5))
    _check(w, router=router, vs_rule=vs_rule)


def test_variable_length_dense_equals_oracle():
    w = Workload("varlen_dense", 2, 2, 1, 128, 1536, 128, lengths=(1536 - 100, 700))
    q, k, v, _ = make_qkv(w)
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lens = torch.tensor(w.lengths, dtype=torch.int32, device="cuda")
    p = C.params_for(qd, kd, block=128, seq_lens=lens)
    ws = C.alloc_workspace(p)
    o, lse = C.crisp_dense_prefill(p, qd, kd, vd, ws)
    assert C.crisp_get_device_status(ws) == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    for b, n in enumerate(w.lengths):
        nb = O.n_blocks(n, 128)
        full = np.tril(np.ones((nb, nb), dtype=bool))
        for h in range(2):
            ref, lref, rows = O.masked_attention_rows(O.bf16_to_f64(q[b, h, :n]), O.bf16_to_f64(k[b, 0, :n]),
                                                      O.bf16_to_f64(v[b, 0, :n]), full, 128, 128 ** -0.5)
            err = np.abs(o[b, h, :n] - ref)
            assert err.max() <= 2e-2 and err.mean() <= 2e-3
            np.testing.assert_allclose(lse[b, h, :n], lref, atol=2e-3)
            assert not o[b, h, n:].any() and np.all(lse[b, h, n:] == -np.inf)


def test_length_out_of_range_is_reported_and_clamped():
    w = Workload("badlen", 2, 2, 1, 64, 1024, 64, lengths=(1024, 1024))
    q, k, v, _ = make_qkv(w)
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lens = torch.tensor([1024, 100], dtype=torch.int32, device="cuda")   # 100 <= 2 * block
    p = C.params_for(qd, kd, block=64, seq_lens=lens)
    ws = C.alloc_workspace(p)
    pattern, score, pv, ps = C.crisp_route(p, qd, kd, ws)
    C.crisp_select(p, qd, kd, pattern, pv, ps, ws)
    assert C.crisp_get_device_status(ws) == -6
    assert C.crisp_get_device_status(ws) == 0


# ---- token-granular vertical-slash masks (slash blocks as diagonal bands)
TOKEN_TINY = Workload("token_tiny", 1, 2, 1, 128, 4096, 128, diffuse_heads=(1,), sink_logit=8.0,
                      n_vertical=2, recency_peak=9.0, recency_freqs="rope")


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.0])
def test_token_granularity_tiny(alpha):
    reps = _check(TOKEN_TINY, alpha=alpha, granularity="token", expect_both=True)
    assert reps[0]["pattern"] == O.VS


@pytest.mark.parametrize("kw", [
    dict(seqlen=4096 + 77, head_dim=128, h_q=4, h_kv=2),                   # ragged, 77-row last block
    dict(seqlen=3 * 128 + 1, head_dim=64, h_q=2, h_kv=1),                  # N_b = 4, one-token last block
    dict(batch=2, seqlen=4096, head_dim=128, h_q=4, h_kv=2, lengths=(3001, 4096)),
])
def test_token_granularity_shapes(kw):
    base = dict(name="token", batch=1, block=128, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    base.update(kw)
    _check(Workload(**base), granularity="token")


def test_token_granularity_llama_32k():
    w = WORKLOADS["llama_32k"]
    reps = _check(w, granularity="token", heads=range(0, 32, 2),
                  qblocks_fn=lambda b, h: PU.sample_qblocks(w.n_blocks, 3, 5000 + h))
    assert {r["pattern"] for r in reps} == {O.VS, O.PE}


def test_kmin_above_nb():
    w = Workload("kmin", 1, 2, 1, 64, 512, 64, diffuse_heads=(1,), n_vertical=0, sink_logit=8.0)
    q, k, v, _ = make_qkv(w)
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = C.params_for(qd, kd, block=64, k_min_blocks=50)
    ws = C.alloc_workspace(p)
    pattern, score, pv, ps = C.crisp_route(p, qd, kd, ws)
    mask, tidx, tcnt = C.crisp_select(p, qd, kd, pattern, pv, ps, ws)
    if int(pattern[0]) == O.VS:      # k_min > N_b clips to N_b: every causal tile
        assert torch.equal(mask[0].cpu().bool(), torch.tril(torch.ones(8, 8, dtype=torch.bool)))


def test_dense_equals_oracle_full_mask():
    w = Workload("dense", 1, 4, 2, 128, 1024, 128, n_vertical=2)
    q, k, v, _ = make_qkv(w)
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = C.params_for(qd, kd, block=128)
    ws = C.alloc_workspace(p)
    o, lse = C.crisp_dense_prefill(p, qd, kd, vd, ws)
    assert C.crisp_get_device_status(ws) == 0
    full = np.tril(np.ones((8, 8), dtype=bool))
    for h in range(4):
        ref, lref, rows = O.masked_attention_rows(O.bf16_to_f64(q[0, h]), O.bf16_to_f64(k[0, h // 2]),
                                                  O.bf16_to_f64(v[0, h // 2]), full, 128, 128 ** -0.5)
        err = np.abs(o[0, h].float().cpu().numpy() - ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3
        np.testing.assert_allclose(lse[0, h].cpu().numpy(), lref, atol=2e-3)


def test_sparse_with_full_lists_equals_dense():
    w = Workload("full", 1, 2, 1, 128, 2048, 128)
    q, k, v, _ = make_qkv(w)
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = C.params_for(qd, kd, block=128)
    ws = C.alloc_workspace(p)
    nb = 16
    tidx = torch.arange(nb, dtype=torch.int32, device="cuda").repeat(2, nb, 1).contiguous()
    tcnt = torch.arange(1, nb + 1, dtype=torch.int32, device="cuda").repeat(2, 1).contiguous()
    o1, l1 = C.crisp_sparse_prefill(p, qd, kd, vd, tidx, tcnt, ws)
    o2, l2 = C.crisp_dense_prefill(p, qd, kd, vd, ws)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_out_of_range_tile_index_is_reported_not_read():
    w = Workload("bad", 1, 1, 1, 128, 1024, 128, diffuse_heads=())
    q, k, v, _ = make_qkv(w)
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = C.params_for(qd, kd, block=128)
    ws = C.alloc_workspace(p)
    nb = 8
    tidx = torch.zeros(1, nb, nb, dtype=torch.int32, device="cuda")
    tidx[0, 3, 1] = 7            # key block 7 is above query block 3: rejected by the kernel
    tcnt = torch.ones(1, nb, dtype=torch.int32, device="cuda")
    tcnt[0, 3] = 2
    C.crisp_sparse_prefill(p, qd, kd, vd, tidx, tcnt, ws)
    assert C.crisp_get_device_status(ws) == -6
    assert C.crisp_get_device_status(ws) == 0     # reading clears it


def test_llama_32k():
    w = WORKLOADS["llama_32k"]
    reps = _check(w, qblocks_fn=lambda b, h: PU.sample_qblocks(w.n_blocks, 4, 1000 + h), expect_both=True)
    vs = [r for r in reps if r["pattern"] == O.VS]
    assert len(vs) == 24
    assert max(r["density"] for r in vs) < 0.2


def test_llama_32k_median_floor():
    w = WORKLOADS["llama_32k"]
    reps = _check(w, vs_rule="alpha_median", qblocks_fn=lambda b, h: PU.sample_qblocks(w.n_blocks, 2, 1500 + h))
    assert sum(r["pattern"] == O.VS for r in reps) == 24


def test_variable_length_llama_32k():
    w = WORKLOADS["llama_32k"].with_(name="llama_32k_varlen", batch=2, lengths=(32768 - 5, 20000 + 37))
    reps = _check(w, qblocks_fn=lambda b, h: PU.sample_qblocks(O.n_blocks(w.length(b), 128), 2, 4000 + h),
                  heads=range(0, 32, 3))
    assert {r["pattern"] for r in reps} == {O.VS, O.PE}


# ---- the large configurations: routing and selection of every head in full;
# attention on the first, the last and 30 random query blocks of every head
def _sample32(nb, base):
    return lambda b, h: PU.sample_qblocks(nb, 30, base + h)


@pytest.mark.slow
def test_qwen_131k_alpha_and_gamma():
    w = WORKLOADS["qwen_131k"]
    _check_alphas(w, (1.0, 1.0), lambda i, h: PU.sample_qblocks(w.n_blocks, 30, 2000 + h), _device_inputs(w),
                  vs_rules=["alpha", "gamma"])


@pytest.mark.slow
def test_llama_512k_alpha_schedule():
    # the headline input at alpha 1 (30 random query blocks per head) and the
    # CRISP page's speed settings alpha 1.25 and 1.5 (Section 5.3; 2 random)
    w = WORKLOADS["llama_512k"]
    nb = w.n_blocks
    reps = _check_alphas(w, (1.0, 1.25, 1.5), lambda i, h: PU.sample_qblocks(nb, 30 if i == 0 else 2, 3000 + h),
                         _device_inputs(w), expect_both=True)
    assert sum(r["pattern"] == O.VS for r in reps[0]) == 24


# ---- sweep points beyond alpha = 1: selection in full, attention sampled
# (at 512k on the first, the last and one random query block per head: at
# alpha = 0.5 every tile is selected and each sampled block costs the oracle
# a full causal row)
@pytest.mark.slow
@pytest.mark.parametrize("seqlen,f", [(65536, 0.0), (65536, 0.5), (524288, 0.0), (524288, 0.5)])
def test_sweep_points_alpha_half_and_two(seqlen, f):
    w = sweep_workload(seqlen, f)
    nb = w.n_blocks
    n_random = 4 if seqlen <= 65536 else 1
    _check_alphas(w, (0.5, 2.0), lambda i, h: PU.sample_qblocks(nb, n_random, 6000 + 31 * i + h),
                  _device_inputs(w), expect_both=f > 0)


# ---- a workload with a RoPE-style recency band (geometric frequencies)
def test_llama_32k_rope_recency():
    w = WORKLOADS["llama_32k_rope"]
    reps = _check(w, qblocks_fn=lambda b, h: PU.sample_qblocks(w.n_blocks, 4, 7000 + h), expect_both=True)
    assert sum(r["pattern"] == O.VS for r in reps) == 24


# ---- the FlexPrefill comparison path at scale (JSD routing, gamma-cumsum VS
# index, Appendix A), as the latency comparison runs it
@pytest.mark.slow
@pytest.mark.parametrize("gamma", [0.95, 0.97])
def test_flexprefill_path_llama_64k(gamma):
    w = sweep_workload(65536, 0.25)
    reps = _check(w, router="jsd", vs_rule="gamma", gamma=gamma, inputs=_device_inputs(w), keep_on_device=True,
                  qblocks_fn=lambda b, h: PU.sample_qblocks(w.n_blocks, 4, 8000 + h))
    assert {r["pattern"] for r in reps} == {O.VS, O.PE}


@pytest.mark.slow
def test_llama_512k_rope_recency_sampled_heads():
    # at 512k the RoPE far field pulls C_struct below tau_proxy, so every head
    # takes the PE path; four heads (one per pair of KV groups), selection in
    # full, attention on the first, the last and two random query blocks
    w = WORKLOADS["llama_512k_rope"]
    heads = (0, 9, 18, 27)
    reps = _check(w, heads=heads, inputs=_device_inputs(w), keep_on_device=True,
                  qblocks_fn=lambda b, h: PU.sample_qblocks(w.n_blocks, 2, 9000 + h))
    assert len(reps) == len(heads)
