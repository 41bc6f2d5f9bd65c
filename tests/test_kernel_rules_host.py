"""Host-side checks of the index arithmetic two kernels derive from the
oracle's definitions (no GPU): the tile builder's bitmask form of the
vertical-slash tile rule, the attention kernel's per-row column window for
token-granular slash bands, and the attention kernel's walk over 128-key
tiles with per-block membership bits. Each is restated here in plain Python
from the kernel's formula and compared with the oracle over many random
aligned and ragged cases, so a wrong shift or sign in the derivation shows
up on the CPU."""
import numpy as np

import oracle as O


def _cases(rng, n_cases):
    for _ in range(n_cases):
        B = int(rng.choice([8, 16, 128]))
        nb = int(rng.integers(3, 40))
        n = (nb - 1) * B + int(rng.integers(1, B + 1))        # aligned or ragged
        s_v = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
        s_s = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
        yield B, nb, n, s_v, s_s


def test_bitmask_slash_rule_matches_oracle_tile_mask():
    # build_tiles_kernel: kb active iff vertical bit, or slash bit jb = kb + c0 + t,
    # c0 = nb-1-qb, t = 0, t = -1 when some row of qb lies past s, t = +1 when s >= 1
    rng = np.random.default_rng(1)
    for B, nb, n, s_v, s_s in _cases(rng, 400):
        V = np.zeros(nb, bool); V[s_v] = True; V[0] = True
        S = np.zeros(nb, bool); S[s_s] = True; S[nb - 1] = True
        s = (n - 1) % B
        want = O.vs_tile_mask(s_v, s_s, nb, n, B)
        bit = lambda j: 0 <= j < nb and S[j]
        for qb in range(nb):
            rows_q = min(B, n - qb * B)
            lo_ext, up, c0 = s - (rows_q - 1) < 0, s >= 1, nb - 1 - qb
            for kb in range(nb):
                on = kb <= qb and (V[kb] or bit(kb + c0) or (lo_ext and bit(kb + c0 - 1))
                                   or (up and bit(kb + c0 + 1)))
                assert on == want[qb, kb], (B, n, qb, kb)


def test_token_band_window_matches_oracle_token_rule():
    # attn_tc_kernel<.., TOKEN>: for a tile that is not a vertical block, row r
    # sees columns [r - s + e B, r - s + e B + B - 1] of the selected slash blocks
    # nb-1-delta+e (e = -1, 0, +1), clipped to the causal limit; e = -1 and +1
    # alone give the band of e = -1 when r > s and of e = +1 otherwise
    rng = np.random.default_rng(2)
    for B, nb, n, s_v, s_s in _cases(rng, 150):
        cols = np.zeros(nb, bool); cols[s_v] = True; cols[0] = True
        slash = np.zeros(nb, bool); slash[s_s] = True; slash[nb - 1] = True
        s = (n - 1) % B
        for qb in range(nb):
            for kb in range(qb + 1):
                if cols[kb]:
                    continue
                f = 0
                for e in (-1, 0, 1):
                    jb = nb - 1 - (qb - kb) + e
                    if 0 <= jb < nb and slash[jb]:
                        f |= 1 << (e + 1)
                for r in range(min(B, n - qb * B)):
                    t = qb * B + r
                    hi = min(t - kb * B, B - 1)
                    a = r - s - B
                    if f == 5:
                        wlo = a if r > s else a + 2 * B
                        whi = wlo + B - 1
                    elif f:
                        first = (f & -f).bit_length() - 1
                        last = f.bit_length() - 1
                        wlo, whi = a + first * B, a + (last + 1) * B - 1
                    else:
                        wlo, whi = 1, 0
                    lo, hi = max(0, wlo), min(hi, whi)
                    for c in range(min(B, n - kb * B)):
                        j = kb * B + c
                        want = j <= t and bool(slash[(j + n - 1 - t) // B])
                        assert (lo <= c <= hi) == want, (B, n, qb, kb, r, c)


def _walk(lists, nb, block, qt, dense):
    # attn_tc_kernel's StepIter for tile-granularity lists (or the dense walk):
    # 128-key tiles kt in ascending order, with bit i*kpu+ks set when query
    # block qb0+i of the 128-row query tile attends key block kt*kpu+ks
    nsub = kpu = 128 // block
    qb0 = qt * nsub
    rows = [qb0 + i for i in range(nsub) if qb0 + i < nb]
    if dense:
        for kt in range(qt + 1):
            yield kt, sum(1 << (i * kpu + ks) for i in range(nsub) for ks in range(kpu)
                          if kt * kpu + ks <= qb0 + i)
        return
    pos = [0] * len(rows)
    while True:
        heads = [lists[qb][pos[i]] // kpu for i, qb in enumerate(rows) if pos[i] < len(lists[qb])]
        if not heads:
            return
        kt, bits = min(heads), 0
        for i, qb in enumerate(rows):
            while pos[i] < len(lists[qb]) and lists[qb][pos[i]] // kpu == kt:
                bits |= 1 << (i * kpu + lists[qb][pos[i]] % kpu)
                pos[i] += 1
        yield kt, bits


def test_tile_walk_covers_exactly_the_mask():
    # the 128-key steps of each 128-row query tile, read back through their
    # membership bits, give exactly the tile mask's pairs (query block, key
    # block) in strictly ascending key tiles, for 64- and 128-wide blocks and
    # for the dense walk (all causal pairs; there the last query tile of an
    # odd N_b at 64-wide blocks also walks for a block past the sequence)
    rng = np.random.default_rng(4)
    for block in (64, 128):
        for _ in range(60):
            nb = int(rng.integers(3, 30))
            n = (nb - 1) * block + int(rng.integers(1, block + 1))
            s_v = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
            s_s = rng.choice(nb, size=int(rng.integers(0, nb)), replace=False)
            for dense in (False, True):
                mask = np.tril(np.ones((nb, nb), bool)) if dense else O.vs_tile_mask(s_v, s_s, nb, n, block)
                lists = [list(np.flatnonzero(mask[qb])) for qb in range(nb)]
                got = np.zeros_like(mask)
                nsub = 128 // block
                for qt in range((nb + nsub - 1) // nsub):
                    kts = []
                    for kt, bits in _walk(lists, nb, block, qt, dense):
                        kts.append(kt)
                        for i in range(nsub):
                            for ks in range(nsub):
                                if bits >> (i * nsub + ks) & 1:
                                    qb, kb = qt * nsub + i, kt * nsub + ks
                                    assert kb <= qb, (block, nb, qt, kt, bits)
                                    if qb >= nb:
                                        # dense walk, 64-wide blocks, odd N_b: the tile's second
                                        # block lies past the sequence; its rows are >= N and
                                        # the kernel never stores them
                                        assert dense and qb * block >= n
                                        continue
                                    got[qb, kb] = True
                    assert kts == sorted(set(kts)), kts
                assert np.array_equal(got, mask), (block, nb, n, dense)
