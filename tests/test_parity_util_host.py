"""The parity harness itself, on CPU: the exemption bands flag exactly the
decisions within 1e-4 of their threshold, the shared-oracle shortcut of the
large configurations equals the plain per-setting oracle, and the tile-list
check accepts the ascending non-zeros of a mask row and nothing else."""
import numpy as np
import pytest
import torch

import oracle as O
import parity_util as PU
from synthetic import WORKLOADS, make_qkv


def _p_with_blocks_at_threshold(nb=20):
    # sink 0.5, local 0.2 and a flat background of 0.3 / 18 per middle block:
    # the mean floor is (1 - 0.7) / 18, so every middle block sits on mu
    p = np.full(nb, 0.0)
    p[0], p[-1] = 0.5, 0.2
    p[1:-1] = 0.3 / (nb - 2)
    return p


def test_vs_exempt_alpha_flags_blocks_on_the_threshold():
    p = _p_with_blocks_at_threshold()
    mu = O.noise_floor(p)
    ex = PU.vs_exempt(p, "alpha", 1.0, 0.95, k_min=2)
    # every middle block equals mu exactly: all of them lie in the band; with
    # them the count above the threshold is ambiguous (2 to 20) around k_min,
    # so the block holding the k_min-th largest value (the local block, 0.2)
    # is exempt too, and only the sink's decision stays exact
    assert ex[1:-1].all()
    assert ex[-1] and not ex[0]
    # lift one block clearly above the floor and lower another clearly below:
    # neither is in the band any more
    q = p.copy()
    q[3] *= 1.5
    q[4] *= 0.5
    ex2 = PU.vs_exempt(q, "alpha", 1.0, 0.95, k_min=2)
    thr = float(np.float32(O.noise_floor(q)))
    assert ex2[3] == (abs(np.float32(q[3]) - thr) <= 1e-4 * thr)
    assert not ex2[4]
    assert float(mu) > 0


def test_vs_exempt_alpha_top_k_fill_band():
    # fewer than k_min blocks pass the threshold: the fill takes the next
    # largest, and blocks tied (within 1e-4) with the k-th value are exempt
    nb = 12
    p = np.array([0.6, 0.1, 0.05, 0.05, 0.05, 0.02, 0.02, 0.02, 0.02, 0.02, 0.02, 0.03])
    p = p / p.sum()
    ex = PU.vs_exempt(p, "alpha", 4.0, 0.95, k_min=5)
    order = np.lexsort((np.arange(nb), -p.astype(np.float32).astype(np.float64)))
    vk = np.float32(p[order[4]])
    want = np.abs(p.astype(np.float32) - vk) <= 1e-4 * vk
    assert (ex & want).sum() == want.sum()
    assert ex[2] and ex[3] and ex[4]                        # the three tied 0.05 blocks


def test_vs_exempt_gamma_flags_the_cut_and_ambiguous_prefix():
    # descending scores whose prefix reaches gamma = 0.95 exactly after four
    # blocks: the cut is ambiguous under rounding, so its neighbours are exempt
    p = np.array([0.5, 0.25, 0.15, 0.05, 0.03, 0.02])
    ex = PU.vs_exempt(p, "gamma", 1.0, 0.95, k_min=1)
    assert ex[3]                                            # the 4th block closes the prefix at 0.95
    assert ex[4]                                            # and the next one could be taken instead
    assert not ex[0]


def test_pe_exempt_flags_ties_at_the_cut():
    nb = 6
    a_bar = np.tril(np.ones((nb, nb)))
    a_bar /= a_bar.sum(axis=1, keepdims=True)               # causal rows summing to one
    ex = PU.pe_exempt(a_bar, 0.95)
    vals = (a_bar / a_bar.sum())[np.tril_indices(nb)]
    # the entries equal to the cut value are all exempt, and they are all in the triangle
    assert ex.sum() >= 1 and not np.triu(ex, 1).any()
    sel = O.pe_index(a_bar, 0.95)
    cut = np.float32((a_bar / a_bar.sum()).flat[sel[-1]])
    tied = np.isclose((a_bar / a_bar.sum()).astype(np.float32), cut, rtol=1e-4, atol=0) & np.tril(
        np.ones((nb, nb), dtype=bool))
    assert (ex | ~tied).all()
    assert vals.size == nb * (nb + 1) // 2


@pytest.mark.parametrize("variants", [
    [("alpha", 1.0), ("alpha", 0.5), ("alpha", 2.0)],
    [("alpha", 1.0), ("gamma", 1.0), ("alpha_median", 1.0)],
])
def test_shared_oracle_equals_the_per_setting_oracle(variants):
    w = WORKLOADS["tiny"]
    q, k, _, _ = make_qkv(w)
    oprms = [PU.oracle_params(w, vs_rule=r, alpha=a) for r, a in variants]
    for h in range(w.h_q):
        qh, kh = O.bf16_to_f64(q[0, h]), O.bf16_to_f64(k[0, 0])
        shared = PU.oracle_for_alphas(qh, kh, oprms)
        for prm, got in zip(oprms, shared):
            want = O.head_route_and_select(qh, kh, prm)
            assert got["pattern"] == want["pattern"]
            np.testing.assert_array_equal(got["mask"], want["mask"])
            if want["pattern"] == O.VS:
                np.testing.assert_array_equal(got["s_v"], want["s_v"])
                np.testing.assert_array_equal(got["s_s"], want["s_s"])


def test_shared_oracle_refuses_settings_that_change_routing_or_the_pe_index():
    w = WORKLOADS["tiny"]
    q, k, _, _ = make_qkv(w)
    qh, kh = O.bf16_to_f64(q[0, 0]), O.bf16_to_f64(k[0, 0])
    with pytest.raises(AssertionError):
        PU.oracle_for_alphas(qh, kh, [PU.oracle_params(w), PU.oracle_params(w, router="jsd")])
    with pytest.raises(AssertionError):
        PU.oracle_for_alphas(qh, kh, [PU.oracle_params(w), PU.oracle_params(w, gamma=0.97)])


def test_list_check_accepts_the_mask_rows_and_rejects_anything_else():
    rng = np.random.default_rng(3)
    bh, nb = 2, 9
    mask = np.tril(rng.random((bh, nb, nb)) < 0.5)
    mask[:, np.arange(nb), np.arange(nb)] = True
    idx = np.zeros((bh, nb, nb), dtype=np.int32)
    cnt = mask.sum(-1).astype(np.int32)
    for b in range(bh):
        for qb in range(nb):
            ids = np.nonzero(mask[b, qb])[0]
            idx[b, qb, :ids.size] = ids
            idx[b, qb, ids.size:] = -7                       # past the count: never read
    m_t, i_t, c_t = torch.from_numpy(mask.astype(np.uint8)), torch.from_numpy(idx), torch.from_numpy(cnt)
    PU.lists_match_mask_on_device(m_t, i_t, c_t)
    bad = i_t.clone()
    bad[1, nb - 1, 0] = nb - 1 if int(bad[1, nb - 1, 0]) != nb - 1 else 0   # a wrong id
    with pytest.raises(AssertionError):
        PU.lists_match_mask_on_device(m_t, bad, c_t)
    worse = c_t.clone()
    worse[0, 4] += 1                                        # a wrong count
    with pytest.raises(AssertionError):
        PU.lists_match_mask_on_device(m_t, i_t, worse)
