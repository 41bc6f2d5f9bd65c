"""Float64 CPU restatement of CRISP sparse prefill (test infrastructure only).

Notation follows the CRISP paper: n keys, head dim d, block size B,
N_b = n / B blocks, representative query block Q_hat = the last b = B query
rows, proxy map A_hat = Softmax(Q_hat K^T / sqrt(d)).

Readings of steps the paper leaves open (each is stated where it is used):
  * A_hat is causal (query row r sits at position n - b + r).
  * blockpool sums the per-key means inside a block, so the block scores of
    each direction sum to one (the only reading under which Eq. 3's
    "1 - p[0] - p[N_b-1]" is a residual mass).
  * the slash (diagonal) index of entry (r, j) is j + (b - 1 - r), the key
    where its diagonal meets the last query row; so slash block 0 is the
    farthest diagonals and slash block N_b-1 the local ones.
  * decisions (route, threshold compare, top-k, gamma cut) are taken on
    float32 values, the kernel's precision; the scores feeding them are
    computed in float64 and rounded once.
  * n need not be a multiple of B: Section 4.3 partitions the map into
    N_b = ceil(n / B) blocks, so the last block holds n - (N_b - 1) B
    tokens. Q_hat is still the last B query rows (Algorithm 2 takes the last
    b rows, a count); block sums and block means run over the tokens a block
    holds; the anchors of Eq. 2 stay the first and last block of the
    partition, so C_struct = p_v[0] + p_v[N_b - 1] as in Algorithm 3.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "VS", "PE", "CrispParams", "bf16_to_f64", "n_blocks", "proxy_attention", "vertical_slash_scores",
    "c_struct_from_map", "route_cstruct", "pooled_estimate_last_block", "js_distance",
    "route_jsd", "noise_floor", "noise_floor_median", "vs_index_alpha", "vs_index_gamma", "pe_pool",
    "pe_estimate", "pe_index", "vs_tile_mask", "vs_tile_mask_tokenwise", "pe_tile_mask",
    "masked_attention_rows", "head_route_and_select", "crisp_prefill",
]

VS, PE = 0, 1


@dataclass
class CrispParams:
    """Hyper-parameters of one CRISP prefill (CRISP paper, Section 5 Setup)."""

    block: int = 128
    alpha: float = 1.0
    gamma: float = 0.95
    tau_proxy: float = 0.2
    tau_jsd: float = 0.1
    k_min_blocks: int = 8
    router: str = "cstruct"   # "cstruct" (Eq. 2) or "jsd" (Appendix A, Algorithm 5)
    vs_rule: str = "alpha"    # "alpha" (Algorithm 3), "alpha_median" (Algorithm 3 with the
                              # median floor of Appendix H) or "gamma" (Appendix A, Algorithm 6)
    granularity: str = "tile" # VS mask of Eq. 1: "tile" (selected blocks as whole tiles) or
                              # "token" (slash blocks as diagonal bands inside the tiles)
    sm_scale: float = 0.0     # 0 -> 1/sqrt(d)

    def scale(self, d: int) -> float:
        return self.sm_scale if self.sm_scale > 0 else 1.0 / math.sqrt(d)


def bf16_to_f64(t) -> np.ndarray:
    """Exact widening of a torch bfloat16 tensor to a float64 numpy array."""
    import torch
    return t.detach().to("cpu").to(torch.float32).numpy().astype(np.float64)


# ---------------------------------------------------------------------------
# (a) Proxy attention — CRISP paper, Algorithm 2 (PatSearch): the proxy map.
# ---------------------------------------------------------------------------
def proxy_attention(q_hat: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """A_hat = Softmax(Q_hat K^T * scale) with causal masking.

    q_hat: [b, d] — the last b query rows (the representative block of Algorithm 2).
    k:     [n, d] — all keys.  Row r of q_hat is at position n - b + r and
    sees keys j <= n - b + r (reading: causal prefill).
    Returns [b, n] float64; masked entries are exactly 0.
    """
    b, n = q_hat.shape[0], k.shape[0]
    logits = (q_hat @ k.T) * scale
    pos = n - b + np.arange(b)
    visible = np.arange(n)[None, :] <= pos[:, None]
    logits = np.where(visible, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=1, keepdims=True)


def n_blocks(n: int, block: int) -> int:
    """N_b = ceil(n / B) (Section 4.3)."""
    return -(-n // block)


def _block_sums(x: np.ndarray, block: int) -> np.ndarray:
    """Sum of x over each block of the N_b = ceil(n / B) partition of axis 0
    (the last block may hold fewer than B entries)."""
    n = x.shape[0]
    nb = n_blocks(n, block)
    pad = np.zeros((nb * block - n,) + x.shape[1:], dtype=x.dtype)
    return np.concatenate([x, pad]).reshape((nb, block) + x.shape[1:]).sum(axis=1)


def vertical_slash_scores(a_hat: np.ndarray, block: int):
    """Block scores p_v (vertical) and p_s (slash) that Algorithm 3 thresholds.

    a_v = colmean(A_hat): mean over the b proxy rows of each key column.
    a_s = diagmean(A_hat): mean over rows of the entries on each diagonal,
    the diagonal of entry (r, j) indexed by j + (b - 1 - r).
    blockpool: sum of the per-key (per-diagonal) means inside each block.
    """
    b, n = a_hat.shape
    a_v = a_hat.mean(axis=0)
    a_s = np.zeros(n)
    for r in range(b):
        shift = b - 1 - r
        a_s[shift:] += a_hat[r, : n - shift]
    a_s /= b
    return _block_sums(a_v, block), _block_sums(a_s, block)


def c_struct_from_map(a_hat: np.ndarray, block: int) -> float:
    """Eq. 2: mean over proxy rows of the mass at the anchor positions.

    Anchors: the sink window (first block) and the local recency window
    (last block); Section 4.3 states these windows are exactly the first and
    last block (reading at B=64: one block, not 128 tokens; for a partial
    last block, that block: keys (N_b - 1) B .. n - 1).
    """
    b, n = a_hat.shape
    anchors = np.zeros(n, dtype=bool)
    anchors[:block] = True
    anchors[(n_blocks(n, block) - 1) * block:] = True
    return float(a_hat[:, anchors].sum() / b)


def route_cstruct(c: float, tau: float) -> int:
    """The routing rule of Algorithm 2 with Eq. 2: VS iff C_struct >= tau_proxy (float32 compare)."""
    return VS if np.float32(c) >= np.float32(tau) else PE


# ---------------------------------------------------------------------------
# JSD router (comparison path) — CRISP paper, Appendix A, Algorithm 5.
# ---------------------------------------------------------------------------
def pooled_estimate_last_block(q_hat: np.ndarray, k: np.ndarray, block: int, scale: float):
    """a_bar = Softmax(pool(Q_hat) pool(K)^T * scale) over all key blocks (Algorithm 5).

    pool = block mean. The last query block sees every key block, so no
    block-level causal mask applies.
    """
    k_bar = pe_pool(k, block)
    q_bar = q_hat.mean(axis=0)
    z = (k_bar @ q_bar) * scale
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def _kl(p: np.ndarray, m: np.ndarray) -> float:
    nz = p > 0
    return float(np.sum(p[nz] * np.log(p[nz] / m[nz])))


def js_distance(a_hat: np.ndarray, a_bar: np.ndarray) -> float:
    """The Jensen-Shannon distance of Algorithm 5: D_JS = sqrt(KL(a_hat||m)/2 + KL(a_bar||m)/2),
    m the mean of the two distributions.

    Natural logarithm; 0*log(0) = 0.
    """
    m = 0.5 * (a_hat + a_bar)
    return math.sqrt(max(0.5 * _kl(a_hat, m) + 0.5 * _kl(a_bar, m), 0.0))


def route_jsd(djs: float, tau: float) -> int:
    """The routing rule of Algorithm 5: VS iff D_JS >= tau (float32 compare)."""
    return VS if np.float32(djs) >= np.float32(tau) else PE


# ---------------------------------------------------------------------------
# (b) Sink-aware vertical-slash selection — Algorithm 3, Eq. 3 and Eq. 4.
# ---------------------------------------------------------------------------
def noise_floor(p: np.ndarray) -> np.float32:
    """Eq. 3: the mean mass of the non-retained blocks, mu = max(1 - p[0] - p[N_b-1], 0) / (N_b - 2)."""
    p32 = p.astype(np.float32)
    nb = p32.shape[0]
    r = np.float32(1.0) - p32[0] - p32[nb - 1]
    r = max(r, np.float32(0.0))
    return np.float32(r / np.float32(nb - 2))


def noise_floor_median(p: np.ndarray) -> np.float32:
    """Appendix H, "Median instead of mean as the noise floor" (Table 9): the
    floor is the median of the non-retained blocks 1..N_b-2 instead of their
    mean, so one dominant block cannot lift it above weaker genuine signal.

    Reading (the page names the statistic only): the textbook median of the
    N_b - 2 float32 scores, i.e. the middle value of the sorted scores, or
    for an even count the mean of the two middle values, (a + b) * 0.5 taken
    in float32.
    """
    mid = np.sort(p.astype(np.float32)[1:-1])
    m = mid.shape[0]
    if m % 2:
        return np.float32(mid[m // 2])
    return np.float32(np.float32(mid[m // 2 - 1] + mid[m // 2]) * np.float32(0.5))


def _topk_desc(values32: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest values; equal values -> lower index first."""
    order = np.lexsort((np.arange(values32.shape[0]), -values32.astype(np.float64)))
    return np.sort(order[:k])


def vs_index_alpha(p: np.ndarray, alpha: float, k_min: int, floor: str = "mean") -> np.ndarray:
    """The sink-aware index of Algorithm 3 (Eq. 3-4) for one direction.

    k_d = #{j : p[j] > alpha * mu} over all blocks (Eq. 4, strict),
    clipped to [k_min, N_b]; S_d = top-k_d(p). Returns sorted block ids.
    mu is the mean floor of Eq. 3, or with floor="median" the median floor
    of Appendix H (Table 9).
    """
    p32 = p.astype(np.float32)
    nb = p32.shape[0]
    mu = noise_floor_median(p) if floor == "median" else noise_floor(p)
    thr = np.float32(np.float32(alpha) * mu)
    k = int(np.count_nonzero(p32 > thr))
    k = min(max(k, k_min), nb)
    return _topk_desc(p32, k)


def _gamma_count(sorted_desc32: np.ndarray, gamma: float) -> int:
    """Smallest k with sum of the first k sorted values >= gamma, else all."""
    cs = np.cumsum(sorted_desc32.astype(np.float64))
    hit = np.nonzero(cs >= np.float64(np.float32(gamma)))[0]
    return int(hit[0]) + 1 if hit.size else int(sorted_desc32.shape[0])


def vs_index_gamma(p: np.ndarray, gamma: float, k_min: int) -> np.ndarray:
    """Appendix A, Algorithm 6, one direction: sort descending, accumulate to gamma.

    p is already normalised (Algorithm 6 divides by the total mass,
    which p_v / p_s carry as 1). Reading: the same k_min floor as
    Algorithm 3, so the two rules differ only in the budget.
    """
    p32 = p.astype(np.float32)
    nb = p32.shape[0]
    order = np.lexsort((np.arange(nb), -p32.astype(np.float64)))
    k = _gamma_count(p32[order], gamma)
    k = min(max(k, k_min), nb)
    return np.sort(order[:k])


# ---------------------------------------------------------------------------
# (c) Pooled estimation for diffuse heads — Algorithm 4 (PE Index).
# ---------------------------------------------------------------------------
def pe_pool(x: np.ndarray, block: int) -> np.ndarray:
    """The block-mean pooling of Algorithm 4 ([n, d] -> [N_b, d]);
    a partial last block is the mean of the rows it holds."""
    n = x.shape[0]
    counts = np.minimum(block, n - block * np.arange(n_blocks(n, block)))
    return _block_sums(x, block) / counts[:, None]


def pe_estimate(q_bar: np.ndarray, k_bar: np.ndarray, scale: float) -> np.ndarray:
    """The pooled estimate of Algorithm 4: A_bar = Softmax(Q_bar K_bar^T * scale).

    Reading: causal at block level (query block i sees key blocks j <= i).
    Returns [N_b, N_b]; entries above the diagonal are 0.
    """
    nb = q_bar.shape[0]
    z = (q_bar @ k_bar.T) * scale
    z = np.where(np.tril(np.ones((nb, nb), dtype=bool)), z, -np.inf)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def pe_index(a_bar: np.ndarray, gamma: float) -> np.ndarray:
    """The gamma cut of Algorithm 4: the smallest set of largest normalised entries
    whose mass reaches gamma.

    Flattening covers the causal (lower-triangle) entries in row-major order;
    flat id = i * N_b + j. Equal values -> lower flat id first.
    Returns the selected flat ids (unsorted = selection order).
    """
    nb = a_bar.shape[0]
    ii, jj = np.tril_indices(nb)
    total = a_bar[ii, jj].sum()
    vals32 = (a_bar[ii, jj] / total).astype(np.float32)
    flat = ii.astype(np.int64) * nb + jj
    order = np.lexsort((flat, -vals32.astype(np.float64)))
    k = _gamma_count(vals32[order], gamma)
    return flat[order[:k]]


# ---------------------------------------------------------------------------
# (d) Tile masks and masked attention — Eq. 1.
# ---------------------------------------------------------------------------
def vs_tile_mask(s_v: Sequence[int], s_s: Sequence[int], nb: int, n: Optional[int] = None,
                 block: Optional[int] = None) -> np.ndarray:
    """Tile (qb, kb) of a VS head is computed iff it holds a selected entry.

    Algorithm 3 returns S_v U S_s U {0, N_b-1}: vertical block ids and slash
    block ids, plus the always-kept first and last block (read as vertical
    block 0 and slash block N_b-1; every reading gives the same tiles).
    Slash block jb covers key-query offsets [ob*B, ob*B + B - 1] with
    ob = N_b - 1 - jb, which meet tile (qb, kb) exactly when qb - kb is ob or
    ob + 1. Tiles are computed whole (plus the causal mask in-tile).

    With n given and not a multiple of B the offsets of a slash block are no
    longer aligned to tiles (see _vs_tile_mask_ragged).
    """
    if n is not None and n != nb * block:
        return _vs_tile_mask_ragged(s_v, s_s, n, block)
    col = np.zeros(nb, dtype=bool)
    col[np.asarray(s_v, dtype=np.int64)] = True
    col[0] = True
    off = np.zeros(nb + 1, dtype=bool)          # off[o]: offset block o selected
    off[nb - 1 - np.asarray(s_s, dtype=np.int64)] = True
    off[0] = True
    qb = np.arange(nb)[:, None]
    kb = np.arange(nb)[None, :]
    dlt = qb - kb
    causal = dlt >= 0
    d0 = np.where(causal, dlt, nb)              # index nb is always False
    d1 = np.where(dlt >= 1, dlt - 1, nb)
    return causal & (col[None, :] | off[d0] | off[d1])


def _vs_tile_mask_ragged(s_v, s_s, n: int, block: int) -> np.ndarray:
    """The VS tile rule for a sequence whose last block is partial.

    Pair (t, j), j <= t, lies on slash index j + n - 1 - t. With
    s = (n - 1) mod B, t = qb B + r and j = kb B + c this is
    (N_b - 1 - delta) B + s + (c - r), delta = qb - kb. Over the pairs of a
    tile, c - r takes every value in [-(R_q - 1), C_k - 1] (R_q, C_k: rows /
    keys of the two blocks) off the diagonal and [-(R_q - 1), 0] on it, so
    the tile meets the consecutive slash blocks
    N_b - 1 - delta + floor((s + v) / B) for v between those bounds: up to
    three of them, where aligned blocks meet two.
    """
    nb = n_blocks(n, block)
    s = (n - 1) % block
    col = np.zeros(nb, dtype=bool)
    col[np.asarray(s_v, dtype=np.int64)] = True
    col[0] = True
    on = np.zeros(nb, dtype=bool)
    on[np.asarray(s_s, dtype=np.int64)] = True
    on[nb - 1] = True
    csum = np.concatenate([[0], np.cumsum(on)])          # csum[i] = #selected in [0, i)
    size = np.minimum(block, n - block * np.arange(nb))
    qb = np.arange(nb)[:, None]
    kb = np.arange(nb)[None, :]
    dlt = qb - kb
    vmin = -(size[:, None] - 1) + 0 * kb
    vmax = np.where(dlt >= 1, size[None, :] - 1 + 0 * qb, 0)
    lo = np.clip(nb - 1 - dlt + np.floor_divide(s + vmin, block), 0, nb)
    hi = np.clip(nb - 1 - dlt + np.floor_divide(s + vmax, block), -1, nb - 1)
    hit = (hi >= lo) & (csum[np.clip(hi + 1, 0, nb)] - csum[np.clip(lo, 0, nb)] > 0)
    return (dlt >= 0) & (col[None, :] | hit)


def vs_tile_mask_tokenwise(s_v, s_s, n: int, block: int) -> np.ndarray:
    """Brute-force definition of the same tile mask, token by token.

    Query t attends key j <= t iff block(j) is a selected vertical block, or
    the slash index n - 1 - (t - j) falls in a selected slash block (with
    vertical 0 and slash N_b-1 always kept). A tile is computed iff any of
    its (t, j) pairs is kept. O(n^2): small n only.
    """
    nb = n_blocks(n, block)
    cols = set(int(x) for x in s_v) | {0}
    slash = set(int(x) for x in s_s) | {nb - 1}
    mask = np.zeros((nb, nb), dtype=bool)
    for t in range(n):
        for j in range(t + 1):
            if (j // block) in cols or ((n - 1 - (t - j)) // block) in slash:
                mask[t // block, j // block] = True
    return mask


def pe_tile_mask(selected_flat: np.ndarray, nb: int) -> np.ndarray:
    """PE tile mask: the Algorithm 4 selection plus, for every query block,
    its diagonal tile and key block 0 (reading: keeps every query row's
    softmax defined; consistent with the always-retained first/last blocks
    of Section 4.3)."""
    mask = np.zeros((nb, nb), dtype=bool)
    mask.flat[np.asarray(selected_flat, dtype=np.int64)] = True
    idx = np.arange(nb)
    mask[idx, idx] = True
    mask[:, 0] = True
    return mask


def masked_attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, tile_mask: np.ndarray,
                          block: int, scale: float, qblocks: Optional[Sequence[int]] = None,
                          vs_tokens: Optional[tuple] = None):
    """Eq. 1: O = Softmax(Q K^T * scale + M_S) V with M_S from whole tiles
    and the causal mask; float64 throughout.

    With vs_tokens = (S_v, S_s) the mask of a VS head is taken at token
    granularity inside those tiles: query t sees key j iff block(j) is a
    selected vertical block (or block 0) or the slash index j + n - 1 - t lies
    in a selected slash block (or block N_b - 1) — Eq. 1's M_S with
    j in S_t read token by token.

    Returns (O [len(rows), d], lse [len(rows)], rows) for the listed query
    blocks (all when None). lse is the natural-log sum of exp of the logits.
    """
    n, d = q.shape
    nb = n_blocks(n, block)
    qbs = list(range(nb)) if qblocks is None else list(qblocks)
    if vs_tokens is not None:
        col_on = np.zeros(nb, dtype=bool)
        col_on[np.asarray(vs_tokens[0], dtype=np.int64)] = True
        col_on[0] = True
        slash_on = np.zeros(nb, dtype=bool)
        slash_on[np.asarray(vs_tokens[1], dtype=np.int64)] = True
        slash_on[nb - 1] = True
    outs, lses, rows = [], [], []
    for qb in qbs:
        kbs = np.nonzero(tile_mask[qb, : qb + 1])[0]
        keys = (kbs[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        keys = keys[keys < n]
        t = np.arange(qb * block, min(qb * block + block, n))
        z = (q[t] @ k[keys].T) * scale
        seen = keys[None, :] <= t[:, None]
        if vs_tokens is not None:
            sl = (keys[None, :] + n - 1 - t[:, None]) // block
            seen &= col_on[keys // block][None, :] | slash_on[np.clip(sl, 0, nb - 1)]
        z = np.where(seen, z, -np.inf)
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        s = e.sum(axis=1, keepdims=True)
        outs.append((e @ v[keys]) / s)
        lses.append((m + np.log(s))[:, 0])
        rows.append(t)
    return np.concatenate(outs), np.concatenate(lses), np.concatenate(rows)


# ---------------------------------------------------------------------------
# Algorithm 1 per head, and the whole prefill.
# ---------------------------------------------------------------------------
def head_route_and_select(q_head: np.ndarray, k_head: np.ndarray, prm: CrispParams,
                          force_pattern: Optional[int] = None) -> Dict[str, object]:
    """Algorithm 1 for one query head: PatSearch, then VSIndex or PEIndex.

    q_head, k_head: float64 [n, d]. ``force_pattern`` overrides the route
    (used to compare later stages on the GPU's route for exempt heads).
    """
    n, d = q_head.shape
    B = prm.block
    nb = n_blocks(n, B)
    scale = prm.scale(d)
    q_hat = q_head[n - B:]
    a_hat = proxy_attention(q_hat, k_head, scale)
    p_v, p_s = vertical_slash_scores(a_hat, B)
    c = c_struct_from_map(a_hat, B)
    out: Dict[str, object] = {"p_v": p_v, "p_s": p_s, "c_struct": c}
    if prm.router == "jsd":
        a_bar = pooled_estimate_last_block(q_hat, k_head, B, scale)
        djs = js_distance(p_v, a_bar)
        out["d_js"] = djs
        pattern = route_jsd(djs, prm.tau_jsd)
        out["score"] = djs
    else:
        pattern = route_cstruct(c, prm.tau_proxy)
        out["score"] = c
    out["routed"] = pattern
    if force_pattern is not None:
        pattern = force_pattern
    out["pattern"] = pattern
    if pattern == VS:
        if prm.vs_rule == "gamma":
            s_v = vs_index_gamma(p_v, prm.gamma, prm.k_min_blocks)
            s_s = vs_index_gamma(p_s, prm.gamma, prm.k_min_blocks)
        elif prm.vs_rule in ("alpha", "alpha_median"):
            floor = "median" if prm.vs_rule == "alpha_median" else "mean"
            s_v = vs_index_alpha(p_v, prm.alpha, prm.k_min_blocks, floor)
            s_s = vs_index_alpha(p_s, prm.alpha, prm.k_min_blocks, floor)
        else:
            raise ValueError(f"unknown vs_rule {prm.vs_rule!r}")
        out["s_v"], out["s_s"] = s_v, s_s
        out["mask"] = vs_tile_mask(s_v, s_s, nb, n, B)
        if prm.granularity == "token":
            out["vs_tokens"] = (s_v, s_s)
    else:
        a_bar = pe_estimate(pe_pool(q_head, B), pe_pool(k_head, B), scale)
        sel = pe_index(a_bar, prm.gamma)
        out["a_bar"] = a_bar
        out["pe_selected"] = sel
        out["mask"] = pe_tile_mask(sel, nb)
    return out


def crisp_prefill(q, k, v, prm: CrispParams, qblocks: Optional[Sequence[int]] = None,
                  heads: Optional[Sequence[int]] = None, force_patterns: Optional[dict] = None,
                  masks: Optional[dict] = None, lengths: Optional[Sequence[int]] = None
                  ) -> Dict[str, object]:
    """Algorithm 1 over a whole [batch, H, n, d] problem (float64 numpy inputs).

    GQA: query head h reads KV head h // (H_q / H_kv). ``masks`` (keyed by
    (batch, head)) replaces the oracle's own tile masks for the attention
    step, so attention can be compared on another implementation's mask.
    ``lengths`` gives each batch element's sequence length (its first
    lengths[b] rows; the rest is padding the method never sees).
    Returns per (batch, head) dicts under "heads" and attention rows.
    """
    bsz, hq, n, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    scale = prm.scale(d)
    res: Dict[str, object] = {"heads": {}, "attn": {}}
    heads = list(range(hq)) if heads is None else list(heads)
    for b in range(bsz):
        nv = n if lengths is None else int(lengths[b])
        for h in heads:
            fp = None if force_patterns is None else force_patterns.get((b, h))
            qh, kh, vh = q[b, h, :nv], k[b, h // g, :nv], v[b, h // g, :nv]
            hr = head_route_and_select(qh, kh, prm, force_pattern=fp)
            res["heads"][(b, h)] = hr
            mask = hr["mask"] if masks is None else masks[(b, h)]
            res["attn"][(b, h)] = masked_attention_rows(qh, kh, vh, mask, prm.block, scale, qblocks,
                                                        hr.get("vs_tokens"))
    return res
