"""Pins of the CPU oracle against facts it does not compute itself.

Each test checks one oracle function against brute force written a second
way, a closed form from the CRISP paper (Appendix C), a hand-computed case
(tests/golden), an invariant, or planted-structure recovery.
"""
import math
import os

import numpy as np

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------- proxy map
def _proxy_bruteforce(q_hat, k, scale):
    b, n = len(q_hat), len(k)
    out = [[0.0] * n for _ in range(b)]
    for r in range(b):
        t = n - b + r
        logits = []
        for j in range(t + 1):
            logits.append(sum(q_hat[r][c] * k[j][c] for c in range(len(k[j]))) * scale)
        mx = max(logits)
        den = sum(math.exp(z - mx) for z in logits)
        for j in range(t + 1):
            out[r][j] = math.exp(logits[j] - mx) / den
    return np.array(out)


def test_proxy_matches_bruteforce():
    rng = _rng(1)
    q_hat = rng.standard_normal((4, 8))
    k = rng.standard_normal((24, 8))
    got = O.proxy_attention(q_hat, k, 0.7)
    want = _proxy_bruteforce(q_hat.tolist(), k.tolist(), 0.7)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_proxy_rows_sum_to_one_and_causal_zeros():
    rng = _rng(2)
    q_hat = rng.standard_normal((16, 8))
    k = rng.standard_normal((64, 8))
    a = O.proxy_attention(q_hat, k, 0.3)
    np.testing.assert_allclose(a.sum(axis=1), 1.0, atol=1e-14)
    for r in range(16):
        assert np.all(a[r, 64 - 16 + r + 1:] == 0.0)
        assert np.all(a[r, : 64 - 16 + r + 1] > 0.0)


def test_appendix_c_background_mass_closed_form():
    """App. C: k signal keys at logit z, n-k background keys at z - Delta give each
    background key mass e^-D / (k + (n-k) e^-D); n = keys visible to the row."""
    n, b, d = 96, 8, 4
    z, delta, sig = 3.0, 2.5, [0, 1, 2, 3, 40, 41]
    q_hat = np.zeros((b, d))
    q_hat[:, 0] = 1.0
    k = np.zeros((n, d))
    k[:, 0] = z - delta
    k[sig, 0] = z
    a = O.proxy_attention(q_hat, k, 1.0)
    for r in range(b):
        nvis = n - b + r + 1
        eps = math.exp(-delta) / (len(sig) + (nvis - len(sig)) * math.exp(-delta))
        bg = [j for j in range(nvis) if j not in sig]
        np.testing.assert_allclose(a[r, bg], eps, rtol=1e-12)
        np.testing.assert_allclose(a[r, sig], eps * math.exp(delta), rtol=1e-12)


# --------------------------------------------------------------------------- block scores
def test_scores_each_sum_to_one():
    rng = _rng(3)
    a = O.proxy_attention(rng.standard_normal((16, 8)), rng.standard_normal((128, 8)), 0.5)
    p_v, p_s = O.vertical_slash_scores(a, 16)
    assert p_v.shape == (8,) and p_s.shape == (8,)
    assert abs(p_v.sum() - 1.0) < 1e-13 and abs(p_s.sum() - 1.0) < 1e-13


def test_slash_equals_vertical_for_single_row():
    """With one proxy row the diagonal index j + (b-1-r) is j itself."""
    rng = _rng(4)
    a = O.proxy_attention(rng.standard_normal((1, 8)), rng.standard_normal((64, 8)), 1.0)
    p_v, p_s = O.vertical_slash_scores(a, 8)
    np.testing.assert_array_equal(p_v, p_s)


def test_slash_scores_bruteforce_diagonal_sums():
    """diagmean written out per diagonal offset o = t - j (slash index n-1-o)."""
    rng = _rng(5)
    b, n, B = 8, 64, 8
    a = O.proxy_attention(rng.standard_normal((b, 4)), rng.standard_normal((n, 4)), 1.0)
    _, p_s = O.vertical_slash_scores(a, B)
    want = np.zeros(n // B)
    for r in range(b):
        t = n - b + r
        for j in range(t + 1):
            o = t - j
            want[(n - 1 - o) // B] += a[r, j] / b
    np.testing.assert_allclose(p_s, want, atol=1e-15)


def test_planted_exact_diagonal_goes_to_its_slash_block():
    """K = Q shifted by delta: all proxy mass on offset delta -> one slash block."""
    n, b, B, delta = 64, 8, 8, 19
    d = n + delta + 1
    q = np.zeros((n, d))
    k = np.zeros((n, d))
    for t in range(n):
        q[t, t] = 30.0
    for j in range(n):
        k[j, j + delta] = 1.0   # q_t . k_j = 30 iff t = j + delta
    a = O.proxy_attention(q[n - b:], k, 1.0)
    p_v, p_s = O.vertical_slash_scores(a, B)
    jb = (n - 1 - delta) // B
    assert p_s[jb] > 0.999
    # the vertical view spreads over the keys t - delta of the b rows
    assert p_v.max() < 0.9


# --------------------------------------------------------------------------- routing
def test_cstruct_equals_anchor_block_scores():
    rng = _rng(6)
    a = O.proxy_attention(rng.standard_normal((16, 8)), rng.standard_normal((160, 8)), 0.9)
    p_v, _ = O.vertical_slash_scores(a, 16)
    assert abs(O.c_struct_from_map(a, 16) - (p_v[0] + p_v[-1])) < 1e-14


def test_cstruct_uniform_head_closed_form():
    """Q = 0: row r spreads evenly over its n-B+r+1 visible keys; anchors hold
    the B sink keys and the r+1 visible keys of the last block."""
    n, B, d = 512, 32, 8
    q_hat = np.zeros((B, d))
    k = _rng(7).standard_normal((n, d))
    c = O.c_struct_from_map(O.proxy_attention(q_hat, k, 1.0), B)
    want = np.mean([(B + r + 1) / (n - B + r + 1) for r in range(B)])
    assert abs(c - want) < 1e-14
    assert O.route_cstruct(c, 0.2) == O.PE


def test_route_threshold_is_inclusive():
    assert O.route_cstruct(0.2, 0.2) == O.VS
    assert O.route_cstruct(np.nextafter(np.float32(0.2), np.float32(0)), 0.2) == O.PE
    assert O.route_jsd(0.1, 0.1) == O.VS


def _golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows.setdefault(key, []).append(vals)
    return rows


def test_jsd_closed_forms():
    g = _golden("jsd_closed_forms.txt")
    a = np.array([0.2, 0.3, 0.5])
    assert O.js_distance(a, a) == 0.0
    d = O.js_distance(np.array([0.5, 0.5, 0, 0]), np.array([0, 0, 0.25, 0.75]))
    assert abs(d - float(g["disjoint"][0][0])) < 1e-15
    assert abs(d - math.sqrt(math.log(2))) < 1e-15
    h = O.js_distance(np.array([1.0, 0.0]), np.array([0.5, 0.5]))
    assert abs(h - float(g["half"][0][0])) < 1e-15


def test_jsd_symmetric_and_bounded():
    rng = _rng(8)
    for _ in range(20):
        x = rng.random(12) ** 3
        y = rng.random(12) ** 3
        x /= x.sum()
        y /= y.sum()
        d1, d2 = O.js_distance(x, y), O.js_distance(y, x)
        assert abs(d1 - d2) < 1e-15
        assert 0.0 <= d1 <= math.sqrt(math.log(2)) + 1e-15


def test_pooled_estimate_bruteforce():
    rng = _rng(9)
    q_hat = rng.standard_normal((4, 3))
    k = rng.standard_normal((12, 3))
    got = O.pooled_estimate_last_block(q_hat, k, 4, 0.5)
    qm = [sum(q_hat[r][c] for r in range(4)) / 4 for c in range(3)]
    z = []
    for kb in range(3):
        km = [sum(k[kb * 4 + i][c] for i in range(4)) / 4 for c in range(3)]
        z.append(0.5 * sum(qm[c] * km[c] for c in range(3)))
    e = [math.exp(x) for x in z]
    np.testing.assert_allclose(got, [x / sum(e) for x in e], atol=1e-15)


# --------------------------------------------------------------------------- selection
def test_alpha_rule_hand_cases():
    g = _golden("alpha_rule_hand.txt")
    p = np.array([float(x) for x in g["p"][0]])
    for vals in g["case"]:
        alpha = float(vals[0].split("=")[1])
        kmin = int(vals[1].split("=")[1])
        want = [int(x) for x in vals[3:]]
        got = O.vs_index_alpha(p, alpha, kmin)
        assert got.tolist() == want, (alpha, kmin, got)
    assert abs(float(O.noise_floor(p)) - 0.0425) < 1e-8


def _golden_vectors(name):
    """Splits a fixture into named vectors: {name: {key: [values, ...]}}."""
    out, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "vector":
                cur = out.setdefault(vals[0], {})
            else:
                cur.setdefault(key, []).append(vals)
    return out


def test_median_floor_hand_cases():
    vecs = _golden_vectors("median_floor_hand.txt")
    assert sorted(vecs) == ["A", "B", "C"]
    for name, g in vecs.items():
        p = np.array([float(x) for x in g["p"][0]])
        fl = dict(kv.split("=") for kv in g["floor"][0])
        assert float(O.noise_floor_median(p)) == float(fl["median"]), name
        assert abs(float(O.noise_floor(p)) - float(fl["mean"])) < 1e-8, name
        for vals in g["case"]:
            kw = dict(kv.split("=") for kv in vals[:3])
            want = [int(x) for x in vals[4:]]
            got = O.vs_index_alpha(p, float(kw["alpha"]), int(kw["k_min"]), kw["rule"])
            assert got.tolist() == want, (name, kw, got)


def test_median_floor_is_numpy_median_of_middle_blocks():
    rng = np.random.default_rng(7)
    for nb in (3, 4, 5, 64, 257, 4096):
        p = rng.dirichlet(np.full(nb, 0.3))
        mid32 = p.astype(np.float32)[1:-1]
        ref = float(np.median(mid32.astype(np.float64)))
        got = float(O.noise_floor_median(p))
        assert abs(got - ref) <= 2 ** -23 * abs(ref) + 1e-45, (nb, got, ref)


def test_median_floor_ignores_anchors_and_outlier_size():
    rng = np.random.default_rng(3)
    p = rng.dirichlet(np.ones(33))
    base = float(O.noise_floor_median(p))
    q = p.copy()
    q[0], q[-1] = 50.0, 70.0                 # the retained blocks do not enter the floor
    assert float(O.noise_floor_median(q)) == base
    # move mass from the sink block into the largest middle block (the scores
    # still sum to one): the median stays, the mean floor of Eq. 3 rises
    q = p.copy()
    j = 1 + int(np.argmax(p[1:-1]))
    d = 0.5 * p[0]
    q[j] += d
    q[0] -= d
    assert float(O.noise_floor_median(q)) == base
    assert float(O.noise_floor(q)) > float(O.noise_floor(p)) + 0.4 * d / 31


def test_median_floor_equals_mean_floor_on_flat_background():
    nb = 18
    p = np.full(nb, 0.5 / (nb - 2))
    p[0], p[-1] = 0.3, 0.2
    assert float(O.noise_floor_median(p)) == float(np.float32(0.5 / 16))
    for a in (0.5, 1.0, 2.0):
        assert (O.vs_index_alpha(p, a, 2, "median").tolist()
                == O.vs_index_alpha(p, a, 2, "mean").tolist())


def test_noise_floor_clamps_at_zero():
    p = np.array([0.7, 0.0, 0.0, 0.4])   # first + last > 1
    assert float(O.noise_floor(p)) == 0.0
    # every block with positive score passes a zero floor
    assert O.vs_index_alpha(p, 1.0, 1).tolist() == [0, 3]


def test_alpha_rule_clips_to_nb():
    p = np.full(6, 1 / 6)
    assert O.vs_index_alpha(p, 0.5, 8).tolist() == list(range(6))


def _failure_vectors():
    nb = 32
    col = np.full(nb, 0.02 / 30)
    col[0], col[7] = 0.96, 0.02
    acc = np.full(nb, 0.295 / 30)
    acc[0], acc[5] = 0.505, 0.2
    return col, acc


def test_gamma_sink_only_collapse_and_noise_accumulation():
    g = _golden("gamma_failure_modes.txt")
    col, acc = _failure_vectors()
    assert len(O.vs_index_gamma(col, 0.95, 1)) == int(g["collapse_gamma_k"][0][0])
    assert 7 not in O.vs_index_gamma(col, 0.95, 1)
    sel = O.vs_index_alpha(col, 1.0, 1)
    assert len(sel) == int(g["collapse_alpha_k"][0][0]) and 7 in sel
    assert len(O.vs_index_gamma(acc, 0.95, 1)) == int(g["accumulate_gamma_k"][0][0])
    assert O.vs_index_alpha(acc, 1.0, 1).tolist() == [0, 5]
    assert len(O.vs_index_alpha(acc, 1.0, 1)) == int(g["accumulate_alpha_k"][0][0])


def test_gamma_noise_count_grows_linearly_with_nb():
    """App. C: the gamma cut collects ~ gamma_residual * n background blocks."""
    counts = []
    for nb in (64, 128, 256, 512):
        p = np.full(nb, 0.3 / (nb - 2))
        p[0], p[1] = 0.5, 0.2
        counts.append(len(O.vs_index_gamma(p, 0.95, 1)) - 2)
        assert len(O.vs_index_alpha(p, 1.0, 1)) == 2
    for nb, c in zip((64, 128, 256, 512), counts):
        assert abs(c - (0.25 / 0.3) * (nb - 2)) <= 1.0


def test_gamma_takes_all_when_total_short():
    p = np.full(10, 0.09)   # total 0.9 < gamma
    assert len(O.vs_index_gamma(p, 0.95, 1)) == 10


def test_gamma_ties_break_to_lower_index():
    p = np.array([0.4, 0.2, 0.2, 0.2])
    assert O.vs_index_gamma(p, 0.75, 1).tolist() == [0, 1, 2]


def test_pe_pool_and_estimate_bruteforce():
    rng = _rng(10)
    x = rng.standard_normal((12, 3))
    pooled = O.pe_pool(x, 4)
    for i in range(3):
        np.testing.assert_allclose(pooled[i], x[4 * i:4 * i + 4].sum(axis=0) / 4, atol=1e-15)
    qb, kb = rng.standard_normal((4, 3)), rng.standard_normal((4, 3))
    a = O.pe_estimate(qb, kb, 0.3)
    for i in range(4):
        z = [0.3 * float(qb[i] @ kb[j]) for j in range(i + 1)]
        e = [math.exp(v) for v in z]
        np.testing.assert_allclose(a[i, : i + 1], [v / sum(e) for v in e], atol=1e-15)
        assert np.all(a[i, i + 1:] == 0)


def test_pe_index_hand_case():
    # rows: [1], [0.7, 0.3], [0.5, 0.3, 0.2]; total 3 -> normalised /3
    a = np.array([[1.0, 0, 0], [0.7, 0.3, 0], [0.5, 0.3, 0.2]])
    # sorted: 1/3 (0,0), 0.7/3 (1,0), 0.5/3 (2,0), 0.3/3 (1,1), 0.3/3 (2,1), 0.2/3 (2,2)
    sel = O.pe_index(a, 0.8)    # cumsum 1/3, 1.7/3, 2.2/3, 2.5/3 >= 0.8 -> 4 entries
    assert sel.tolist() == [0, 3, 6, 4]
    m = O.pe_tile_mask(sel, 3)
    assert m.tolist() == [[1, 0, 0], [1, 1, 0], [1, 0, 1]]


def test_vs_tile_mask_matches_tokenwise_definition():
    rng = _rng(11)
    for trial in range(12):
        B, nb = 4, int(rng.integers(3, 12))
        n = nb * B
        s_v = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
        s_s = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
        a = O.vs_tile_mask(s_v, s_s, nb)
        b = O.vs_tile_mask_tokenwise(s_v, s_s, n, B)
        np.testing.assert_array_equal(a, b)


# --------------------------------------------------------------------------- ragged n
# Section 4.3 partitions the map into N_b = ceil(n / B) blocks; the pins below
# take n that is not a multiple of B (partial last block).
RAGGED_N = [(8, 3 * 8 + 1), (8, 5 * 8 + 3), (8, 6 * 8 + 7), (4, 7 * 4 + 2), (16, 4 * 16 + 9)]


def test_ragged_block_scores_bruteforce():
    rng = _rng(21)
    for B, n in RAGGED_N:
        nb = -(-n // B)
        assert O.n_blocks(n, B) == nb
        q_hat, k = rng.standard_normal((B, 4)), rng.standard_normal((n, 4))
        a = _proxy_bruteforce(q_hat.tolist(), k.tolist(), 0.8)
        want_v, want_s = [0.0] * nb, [0.0] * nb
        for r in range(B):
            t = n - B + r
            for j in range(t + 1):
                want_v[j // B] += a[r][j] / B
                want_s[(n - 1 - (t - j)) // B] += a[r][j] / B
        p_v, p_s = O.vertical_slash_scores(O.proxy_attention(q_hat, k, 0.8), B)
        assert p_v.shape == (nb,) and p_s.shape == (nb,)
        np.testing.assert_allclose(p_v, want_v, atol=1e-14)
        np.testing.assert_allclose(p_s, want_s, atol=1e-14)
        np.testing.assert_allclose([p_v.sum(), p_s.sum()], [1.0, 1.0], atol=1e-13)
        # the anchors of Eq. 2 are the first block and the (partial) last block
        c = O.c_struct_from_map(O.proxy_attention(q_hat, k, 0.8), B)
        last = sum(a[r][j] for r in range(B) for j in range((nb - 1) * B, n)) / B
        first = sum(a[r][j] for r in range(B) for j in range(B)) / B
        assert abs(c - (first + last)) < 1e-13


def test_ragged_pooled_estimate_bruteforce():
    # The block means of Algorithm 5 on a partial last block: the block means of K run over
    # the keys each block holds; the estimate is a softmax over all N_b blocks
    rng = _rng(27)
    B, n, d = 8, 8 * 5 + 3, 4
    q_hat, k = rng.standard_normal((B, d)), rng.standard_normal((n, d))
    qm = [sum(q_hat[r][c] for r in range(B)) / B for c in range(d)]
    blocks = [list(range(i, min(i + B, n))) for i in range(0, n, B)]
    kbar = [[sum(k[j][c] for j in blk) / len(blk) for c in range(d)] for blk in blocks]
    z = [0.6 * sum(qm[c] * kb[c] for c in range(d)) for kb in kbar]
    e = [math.exp(x - max(z)) for x in z]
    want = [x / sum(e) for x in e]
    np.testing.assert_allclose(O.pooled_estimate_last_block(q_hat, k, B, 0.6), want, atol=1e-14)


def test_ragged_pooling_means_partial_block():
    x = np.arange(22, dtype=np.float64).reshape(11, 2)        # 11 rows, B = 4: 4 + 4 + 3
    pooled = O.pe_pool(x, 4)
    assert pooled.shape == (3, 2)
    np.testing.assert_array_equal(pooled[2], [(16 + 18 + 20) / 3, (17 + 19 + 21) / 3])
    np.testing.assert_array_equal(pooled[0], [3.0, 4.0])


def test_ragged_vs_tile_mask_matches_tokenwise_definition():
    rng = _rng(22)
    for B in (4, 8):
        for n in [B * m + s for m in (3, 4, 7) for s in range(1, B)]:
            nb = -(-n // B)
            for _ in range(4):
                s_v = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
                s_s = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
                a = O.vs_tile_mask(s_v, s_s, nb, n, B)
                b = O.vs_tile_mask_tokenwise(s_v, s_s, n, B)
                np.testing.assert_array_equal(a, b, err_msg=f"B={B} n={n}")


def test_ragged_slash_block_can_meet_three_tile_diagonals():
    # n = 8*8 + 3 (B = 8): slash block 3 holds slash indices 24..31, i.e. query-key
    # offsets n-1-j* = 35..42, which tiles on diagonals 4 ([25, 39]), 5 ([33, 47])
    # and 6 ([41, 55]) all contain; with n a multiple of B it would meet two.
    B, n, nb = 8, 67, 9
    m = O.vs_tile_mask([], [3], nb, n, B)
    diags = sorted({qb - kb for qb in range(nb) for kb in range(1, qb + 1) if m[qb, kb] and qb - kb > 1})
    assert diags == [4, 5, 6], diags
    m2 = O.vs_tile_mask([], [3], 8, 64, B)
    diags2 = sorted({qb - kb for qb in range(8) for kb in range(1, qb + 1) if m2[qb, kb] and qb - kb > 1})
    assert diags2 == [4, 5], diags2


# --------------------------------------------------------------------------- attention
def _attention_bruteforce(q, k, v, allowed, scale):
    n, d = len(q), len(q[0])
    out, lse = [], []
    for t in range(n):
        z = [(j, sum(q[t][c] * k[j][c] for c in range(d)) * scale) for j in range(n) if allowed(t, j)]
        mx = max(x for _, x in z)
        w = [(j, math.exp(x - mx)) for j, x in z]
        s = sum(x for _, x in w)
        out.append([sum(x * v[j][c] for j, x in w) / s for c in range(d)])
        lse.append(mx + math.log(s))
    return np.array(out), np.array(lse)


def test_masked_attention_bruteforce():
    rng = _rng(12)
    n, d, B = 32, 4, 8
    q, k, v = rng.standard_normal((3, n, d))
    mask = rng.random((4, 4)) < 0.5
    np.fill_diagonal(mask, True)
    o, lse, rows = O.masked_attention_rows(q, k, v, mask, B, 0.6)
    want_o, want_lse = _attention_bruteforce(q.tolist(), k.tolist(), v.tolist(),
                                             lambda t, j: j <= t and mask[t // B, j // B], 0.6)
    np.testing.assert_allclose(o, want_o, atol=1e-13)
    np.testing.assert_allclose(lse, want_lse, atol=1e-13)
    assert rows.tolist() == list(range(n))


def test_full_mask_equals_dense_causal_softmax():
    rng = _rng(13)
    n, d, B = 48, 6, 8
    q, k, v = rng.standard_normal((3, n, d))
    full = np.tril(np.ones((6, 6), dtype=bool))
    o, _, _ = O.masked_attention_rows(q, k, v, full, B, 0.4)
    z = q @ k.T * 0.4 + np.triu(np.full((n, n), -np.inf), 1)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
    np.testing.assert_allclose(o, p @ v, atol=1e-13)


def test_ragged_full_mask_equals_dense_causal_softmax():
    rng = _rng(23)
    B = 8
    for n in (27, 33, 47):
        q, k, v = rng.standard_normal((3, n, 5))
        nb = -(-n // B)
        o, lse, rows = O.masked_attention_rows(q, k, v, np.tril(np.ones((nb, nb), dtype=bool)), B, 0.5)
        want_o, want_lse = _attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), lambda t, j: j <= t, 0.5)
        assert rows.tolist() == list(range(n))
        np.testing.assert_allclose(o, want_o, atol=1e-13)
        np.testing.assert_allclose(lse, want_lse, atol=1e-13)


def test_token_granular_vs_mask_bruteforce():
    # Eq. 1 with S_t read token by token: vertical blocks whole, slash blocks as
    # diagonal bands; aligned and ragged n
    rng = _rng(25)
    B = 8
    for n in (40, 43, 57):
        nb = -(-n // B)
        q, k, v = rng.standard_normal((3, n, 4))
        s_v = rng.choice(nb, size=2, replace=False)
        s_s = rng.choice(nb, size=2, replace=False)
        cols = set(int(x) for x in s_v) | {0}
        slash = set(int(x) for x in s_s) | {nb - 1}
        tiles = O.vs_tile_mask(s_v, s_s, nb, n, B)
        o, lse, _ = O.masked_attention_rows(q, k, v, tiles, B, 0.5, vs_tokens=(s_v, s_s))
        allowed = lambda t, j: j <= t and (j // B in cols or (j + n - 1 - t) // B in slash)
        want_o, want_lse = _attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), allowed, 0.5)
        np.testing.assert_allclose(o, want_o, atol=1e-13)
        np.testing.assert_allclose(lse, want_lse, atol=1e-13)
        # whole tiles see a superset of keys: the token-level lse is never larger
        _, lse_tile, _ = O.masked_attention_rows(q, k, v, tiles, B, 0.5)
        assert np.all(lse <= lse_tile + 1e-12)


def test_token_granular_equals_tiles_when_every_slash_block_is_kept():
    rng = _rng(26)
    B, n = 8, 45
    nb = -(-n // B)
    q, k, v = rng.standard_normal((3, n, 4))
    every = np.arange(nb)
    tiles = O.vs_tile_mask([3], every, nb, n, B)
    a = O.masked_attention_rows(q, k, v, tiles, B, 0.7, vs_tokens=([3], every))
    b = O.masked_attention_rows(q, k, v, tiles, B, 0.7)
    np.testing.assert_allclose(a[0], b[0], atol=1e-14)


def test_prefill_lengths_ignore_padding():
    rng = _rng(24)
    B, N = 8, 48
    q, k, v = rng.standard_normal((3, 2, 2, N, 4))
    lengths = [41, 30]
    prm = O.CrispParams(block=B, k_min_blocks=1)
    res = O.crisp_prefill(q, k, v, prm, lengths=lengths)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for b, nv in enumerate(lengths):               # padding rows change: nothing else may
        q2[b, :, nv:] = 1e3
        k2[b, :, nv:] = -1e3
        v2[b, :, nv:] = 7.0
    res2 = O.crisp_prefill(q2, k2, v2, prm, lengths=lengths)
    for key, hr in res["heads"].items():
        np.testing.assert_array_equal(hr["mask"], res2["heads"][key]["mask"])
        np.testing.assert_array_equal(res["attn"][key][0], res2["attn"][key][0])
        assert res["attn"][key][0].shape[0] == lengths[key[0]]


def test_attention_is_causal():
    rng = _rng(14)
    n, d, B = 40, 4, 8
    q, k, v = rng.standard_normal((3, n, d))
    full = np.tril(np.ones((5, 5), dtype=bool))
    o1, _, _ = O.masked_attention_rows(q, k, v, full, B, 0.5)
    k2, v2 = k.copy(), v.copy()
    k2[21:] += 5.0
    v2[21:] -= 3.0
    o2, _, _ = O.masked_attention_rows(q, k2, v2, full, B, 0.5)
    np.testing.assert_array_equal(o1[:21], o2[:21])
    assert not np.allclose(o1[21:], o2[21:])


# --------------------------------------------------------------------------- planted recovery
def test_planted_recovery_tiny_workload():
    from synthetic import WORKLOADS, make_qkv
    w = WORKLOADS["tiny"]
    q, k, v, meta = make_qkv(w)
    prm = O.CrispParams(block=w.block, alpha=1.0)
    k0 = O.bf16_to_f64(k[0, 0])
    h0 = O.head_route_and_select(O.bf16_to_f64(q[0, 0]), k0, prm)
    h1 = O.head_route_and_select(O.bf16_to_f64(q[0, 1]), k0, prm)
    assert h0["pattern"] == O.VS and h1["pattern"] == O.PE
    assert 0 in h0["s_v"]                       # sink block
    assert w.n_blocks - 1 in h0["s_s"]          # local diagonal block
    assert h0["c_struct"] > 0.5 > 0.2 > h1["c_struct"]
    assert h0["mask"].sum() < h1["mask"].sum()
    # Appendix F: a diffuse (PE) head does not reach gamma within its top 50 blocks
    assert len(h1["pe_selected"]) > 50


def test_alpha_rule_is_sink_aware():
    # Section 4.3: the floor excludes the anchors, so it falls as the sink grows;
    # moving mass from the middle blocks into the sink (scaling them all by c)
    # lowers mu by the same factor and leaves the selected middle blocks unchanged
    rng = _rng(28)
    nb = 24
    p = rng.dirichlet(np.full(nb, 0.4))
    base = O.vs_index_alpha(p, 1.0, 2)
    mu = float(O.noise_floor(p))
    for c in (0.8, 0.5, 0.2):
        q = p.copy()
        q[1:-1] *= c
        q[0] += (1 - c) * p[1:-1].sum()
        assert float(O.noise_floor(q)) < mu
        assert abs(float(O.noise_floor(q)) - c * mu) < 1e-6 * mu
        got = O.vs_index_alpha(q, 1.0, 2)
        assert set(got.tolist()) - {0} == set(base.tolist()) - {0}, c


def test_planted_recovery_verticals_and_jsd_agreement():
    from synthetic import Workload, make_qkv
    w = Workload("small", 1, 4, 1, 128, 8192, 128, diffuse_heads=(3,))
    q, k, v, meta = make_qkv(w)
    kk = O.bf16_to_f64(k[0, 0])
    vert_blocks = sorted({p // w.block for p in meta["verticals"][0]})
    for h in range(4):
        qq = O.bf16_to_f64(q[0, h])
        hr = O.head_route_and_select(qq, kk, O.CrispParams(block=128))
        hj = O.head_route_and_select(qq, kk, O.CrispParams(block=128, router="jsd"))
        assert hr["pattern"] == hj["pattern"]
        if h == 3:
            assert hr["pattern"] == O.PE
        else:
            assert hr["pattern"] == O.VS
            assert set(vert_blocks) <= set(hr["s_v"].tolist())
            assert 0 in hr["s_v"].tolist()
            # the noise floor keeps the flat background out: only the planted
            # columns, the anchors and the k_min fill are selected
            assert len(hr["s_v"]) <= max(8, len(vert_blocks) + 2)
