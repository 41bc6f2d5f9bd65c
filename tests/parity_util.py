"""GPU-vs-oracle comparison with the exemption protocol.

Decisions are compared exactly except for items whose oracle score lies
within EXEMPT_REL (1e-4) relative of the threshold that decides them
(counted and returned); attention is compared against the oracle run on the
GPU's own tile mask: max-abs <= 2e-2 and mean-abs <= 2e-3.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np
import torch

import oracle as O

EXEMPT_REL = 1e-4
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3


def lists_match_mask_on_device(mask, tile_idx, tile_cnt):
    """Tile lists must hold, per query block, the ascending key blocks of its
    mask row: checked with torch on the device, one head at a time (at 512k
    the lists are 2 GiB, too large to bring to the host for every config)."""
    nb = mask.shape[-1]
    cols = torch.arange(nb, device=mask.device, dtype=torch.int32)
    for bh in range(mask.shape[0]):
        m = mask[bh].bool()
        assert torch.equal(m.sum(-1, dtype=torch.int32), tile_cnt[bh]), bh
        pos = (torch.cumsum(m.to(torch.int32), dim=-1) - 1).clamp_(min=0).long()
        got = torch.gather(tile_idx[bh], -1, pos)
        assert torch.equal(got[m], cols.expand(nb, nb)[m]), bh


def run_gpu(w, q, k, v, router="cstruct", vs_rule="alpha", alpha=1.0, gamma=0.95, tau_jsd=0.1,
            granularity="tile", keep_on_device=False):
    """Runs route -> select -> sparse prefill through the C ABI; returns CPU
    copies. With keep_on_device the tile lists are checked against the mask
    on the device and dropped, and o / lse stay on the device (compare_head
    then brings only the compared rows to the host)."""
    import dynamic_block_sparse_qk_b200 as C
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lens = None if w.lengths is None else torch.tensor(list(w.lengths), dtype=torch.int32, device=qd.device)
    p = C.params_for(qd, kd, block=w.block, alpha=alpha, gamma=gamma, router=router,
                     vs_rule=vs_rule, tau_jsd=tau_jsd, seq_lens=lens, granularity=granularity)
    ws = C.alloc_workspace(p, qd.device)
    pattern, score, p_v, p_s = C.crisp_route(p, qd, kd, ws)
    nb = p.n_blocks
    vs_sel = torch.empty(p.batch * p.h_q, 2, nb, dtype=torch.uint8, device=qd.device)
    mask, tidx, tcnt = C.crisp_select(p, qd, kd, pattern, p_v, p_s, ws, want_mask=True, vs_sel=vs_sel)
    o, lse = C.crisp_sparse_prefill(p, qd, kd, vd, tidx, tcnt, ws)
    status = C.crisp_get_device_status(ws)
    out = {"pattern": pattern, "score": score, "p_v": p_v, "p_s": p_s, "vs_sel": vs_sel,
           "mask": mask, "tile_idx": tidx, "tile_cnt": tcnt, "o": o, "lse": lse}
    if keep_on_device:
        assert granularity == "tile"
        lists_match_mask_on_device(mask, tidx, tcnt)
        dev = {"o": o, "lse": lse}
        out = {key: val.cpu() for key, val in out.items() if key not in ("o", "lse", "tile_idx")}
        out.update(dev)
        out["lists_checked"] = True
        del tidx
    else:
        out = {key: val.cpu() for key, val in out.items()}
    out["status"] = status
    out["params"] = p
    del qd, kd, vd, ws, lens
    torch.cuda.empty_cache()
    return out


def oracle_params(w, router="cstruct", vs_rule="alpha", alpha=1.0, gamma=0.95, tau_jsd=0.1,
                  granularity="tile"):
    return O.CrispParams(block=w.block, alpha=alpha, gamma=gamma, router=router, vs_rule=vs_rule,
                         tau_jsd=tau_jsd, granularity=granularity)


TILE_ID_MASK, TILE_WHOLE, TILE_SLASH_SHIFT = 0xFFFFFF, 1 << 24, 25


def expected_token_flags(qb, kb, nb, vs, sel_v, sel_s):
    """Flags a token-granularity list entry must carry (from the GPU's own selection)."""
    if not vs or kb == 0 or sel_v[kb]:
        return TILE_WHOLE
    f = 0
    for e in (-1, 0, 1):
        jb = nb - 1 - (qb - kb) + e
        if jb == nb - 1 or (0 <= jb < nb and sel_s[jb]):
            f |= 1 << (TILE_SLASH_SHIFT + e + 1)
    return f


def _near(x, ref):
    return abs(float(x) - float(ref)) <= EXEMPT_REL * abs(float(ref))


def vs_exempt(p: np.ndarray, rule: str, alpha: float, gamma: float, k_min: int) -> np.ndarray:
    """Blocks whose selection could flip under float rounding (one direction)."""
    p32 = p.astype(np.float32)
    nb = p32.shape[0]
    order = np.lexsort((np.arange(nb), -p32.astype(np.float64)))
    ex = np.zeros(nb, dtype=bool)
    if rule in ("alpha", "alpha_median"):
        mu = O.noise_floor_median(p) if rule == "alpha_median" else O.noise_floor(p)
        thr = np.float32(np.float32(alpha) * mu)
        ex |= np.abs(p32 - thr) <= EXEMPT_REL * abs(thr)
        cnt = int(np.count_nonzero(p32 > thr))
        if cnt < k_min + int(ex.sum()) and k_min <= nb:
            vk = p32[order[min(k_min, nb) - 1]]
            ex |= np.abs(p32 - vk) <= EXEMPT_REL * abs(vk)
    else:
        cs = np.cumsum(p32[order].astype(np.float64))
        g = np.float64(np.float32(gamma))
        hit = np.nonzero(cs >= g)[0]
        kstar = int(hit[0]) + 1 if hit.size else nb
        k = min(max(kstar, k_min), nb)
        vk = p32[order[k - 1]]
        ex |= np.abs(p32 - vk) <= EXEMPT_REL * abs(vk)
        if kstar >= k_min:
            amb = np.nonzero(np.abs(cs - g) <= EXEMPT_REL * g)[0]
            for i in amb:
                for j in (i - 1, i, i + 1, i + 2):
                    if 0 <= j < nb:
                        ex[order[j]] = True
    return ex


def pe_exempt(a_bar: np.ndarray, gamma: float) -> np.ndarray:
    """Tiles of a PE head whose selection could flip under float rounding."""
    nb = a_bar.shape[0]
    ii, jj = np.tril_indices(nb)
    vals = a_bar[ii, jj]
    vals32 = (vals / vals.sum()).astype(np.float32)
    flat = ii.astype(np.int64) * nb + jj
    order = np.lexsort((flat, -vals32.astype(np.float64)))
    cs = np.cumsum(vals32[order].astype(np.float64))
    g = np.float64(np.float32(gamma))
    hit = np.nonzero(cs >= g)[0]
    ex = np.zeros((nb, nb), dtype=bool)
    if not hit.size:
        return ex
    kstar = int(hit[0]) + 1
    vk = vals32[order[kstar - 1]]
    near = np.abs(vals32 - vk) <= EXEMPT_REL * abs(vk)
    ex.flat[flat[near]] = True
    amb = np.nonzero(np.abs(cs - g) <= EXEMPT_REL * g)[0]
    for i in amb:
        for j in (i - 1, i, i + 1, i + 2):
            if 0 <= j < len(order):
                ex.flat[flat[order[j]]] = True
    return ex


def oracle_for_alphas(q_head, k_head, oprms):
    """Oracle results for parameter sets that differ only in their VS index
    (alpha, or the alpha / median / gamma rule at one gamma and router):
    routing and the PE index (which none of those enter) once, then the VS
    index (Algorithm 3, or Algorithm 6 for the gamma rule) and its tile mask
    per set, with the same oracle functions head_route_and_select composes."""
    base = O.head_route_and_select(q_head, k_head, oprms[0])
    outs = [base]
    n = q_head.shape[0]
    p0 = oprms[0]
    for prm in oprms[1:]:
        assert (prm.block, prm.gamma, prm.router, prm.tau_proxy, prm.tau_jsd, prm.granularity) == \
            (p0.block, p0.gamma, p0.router, p0.tau_proxy, p0.tau_jsd, p0.granularity)
        r = dict(base)
        if base["pattern"] == O.VS:
            if prm.vs_rule == "gamma":
                r["s_v"] = O.vs_index_gamma(base["p_v"], prm.gamma, prm.k_min_blocks)
                r["s_s"] = O.vs_index_gamma(base["p_s"], prm.gamma, prm.k_min_blocks)
            else:
                floor = "median" if prm.vs_rule == "alpha_median" else "mean"
                r["s_v"] = O.vs_index_alpha(base["p_v"], prm.alpha, prm.k_min_blocks, floor)
                r["s_s"] = O.vs_index_alpha(base["p_s"], prm.alpha, prm.k_min_blocks, floor)
            r["mask"] = O.vs_tile_mask(r["s_v"], r["s_s"], O.n_blocks(n, prm.block), n, prm.block)
        outs.append(r)
    return outs


def compare_head(gpu, b, h, q_head, k_head, v_head, w, oprm, qblocks=None, score_tol=2e-5, orc=None):
    """Compares one query head; returns a report dict (asserts on hard failures).
    ``orc``: the oracle's result for this head and oprm when already computed."""
    bh = b * w.h_q + h
    n = q_head.shape[0]                        # this sequence's length
    nb = O.n_blocks(n, w.block)                # its blocks; GPU arrays are w.n_blocks wide
    rep = {"head": (b, h), "exempt_route": False, "exempt_blocks": 0, "exempt_differing": 0,
           "route_differs": False}
    if orc is None:
        orc = O.head_route_and_select(q_head, k_head, oprm)
    gp = int(gpu["pattern"][bh])
    # (1) block scores (zero past the sequence's own blocks)
    for key in ("p_v", "p_s"):
        row = gpu[key][bh].double().numpy()
        np.testing.assert_allclose(row[:nb], orc[key], rtol=score_tol, atol=1e-9)
        assert not row[nb:].any(), key
    # (2) route
    tau = oprm.tau_jsd if oprm.router == "jsd" else oprm.tau_proxy
    np.testing.assert_allclose(float(gpu["score"][bh]), orc["score"], rtol=score_tol, atol=1e-7)
    if _near(orc["score"], tau):
        rep["exempt_route"] = True
        if gp != orc["routed"]:
            rep["route_differs"] = True
            orc = O.head_route_and_select(q_head, k_head, oprm, force_pattern=gp)
    else:
        assert gp == orc["routed"], (b, h, gp, orc["routed"], orc["score"])
    rep["pattern"] = gp
    full_mask = gpu["mask"][bh].numpy().astype(bool)
    assert not full_mask[nb:].any() and not full_mask[:, nb:].any()
    gmask = full_mask[:nb, :nb]
    # (3) selection
    if gp == O.VS:
        sel_full = gpu["vs_sel"][bh].numpy().astype(bool)
        assert not sel_full[:, nb:].any()
        sel = sel_full[:, :nb]
        for d, (key, pd) in enumerate((("s_v", orc["p_v"]), ("s_s", orc["p_s"]))):
            want = np.zeros(nb, dtype=bool)
            want[orc[key]] = True
            ex = vs_exempt(pd, oprm.vs_rule, oprm.alpha, oprm.gamma, oprm.k_min_blocks)
            bad = (sel[d] != want) & ~ex
            assert not bad.any(), (b, h, key, np.nonzero(bad)[0][:10])
            rep["exempt_blocks"] += int(ex.sum())
            rep["exempt_differing"] += int(((sel[d] != want) & ex).sum())
        s_v = np.nonzero(sel[0])[0]
        s_s = np.nonzero(sel[1])[0]
        np.testing.assert_array_equal(gmask, O.vs_tile_mask(s_v, s_s, nb, n, w.block))
    else:
        ex = pe_exempt(orc["a_bar"], oprm.gamma)
        want = orc["mask"]
        bad = (gmask != want) & ~ex
        assert not bad.any(), (b, h, np.argwhere(bad)[:10])
        rep["exempt_differing"] += int(((gmask != want) & ex).sum())
        idx = np.arange(nb)
        assert gmask[idx, idx].all() and gmask[:, 0].all()
        assert not np.triu(gmask, 1).any()
        rep["exempt_blocks"] += int(ex.sum())
    # (4) tile lists = ascending nonzeros of the mask row
    cnt_full = gpu["tile_cnt"][bh].numpy()
    assert not cnt_full[nb:].any()
    cnt = cnt_full[:nb]
    np.testing.assert_array_equal(cnt, gmask.sum(axis=1))
    token = oprm.granularity == "token"
    vs_tokens = None
    if token and gp == O.VS:
        vs_tokens = (np.nonzero(sel[0])[0], np.nonzero(sel[1])[0])
    tidx = None if gpu.get("lists_checked") else gpu["tile_idx"][bh].numpy()
    for qb in (range(nb) if tidx is not None else ()):
        ids = tidx[qb, : cnt[qb]]
        if token:
            flags = ids & ~TILE_ID_MASK
            ids = ids & TILE_ID_MASK
            want = [expected_token_flags(qb, int(kb), nb, gp == O.VS, sel[0] if gp == O.VS else None,
                                         sel[1] if gp == O.VS else None) for kb in ids]
            np.testing.assert_array_equal(flags, want)
        np.testing.assert_array_equal(ids, np.nonzero(gmask[qb])[0])
    rep["density"] = float(gmask.sum()) / (nb * (nb + 1) / 2)
    rep["qblocks"] = nb if qblocks is None else len(qblocks)
    # (5) attention on the GPU's own mask
    o_ref, lse_ref, rows = O.masked_attention_rows(q_head, k_head, v_head, gmask, w.block,
                                                   oprm.scale(q_head.shape[1]), qblocks, vs_tokens)
    o_all, lse_all = gpu["o"][b, h], gpu["lse"][b, h]            # host or device tensors
    assert not o_all[n:].any() and bool(torch.all(lse_all[n:] == -float("inf")))     # padding rows
    sel_rows = torch.as_tensor(rows, dtype=torch.long, device=o_all.device)
    o_gpu = o_all[sel_rows].float().cpu().numpy()
    lse_gpu = lse_all[sel_rows].cpu().numpy()
    err = np.abs(o_gpu - o_ref)
    rep["attn_max_abs"] = float(err.max())
    rep["attn_mean_abs"] = float(err.mean())
    rep["attn_rel"] = float(err.max() / max(np.abs(o_ref).max(), 1e-30))
    assert rep["attn_max_abs"] <= ATTN_MAX_ABS and rep["attn_mean_abs"] <= ATTN_MEAN_ABS, rep
    np.testing.assert_allclose(lse_gpu, lse_ref, atol=2e-3, rtol=0)
    return rep


def sample_qblocks(nb: int, n_random: int, seed: int) -> Sequence[int]:
    rng = np.random.default_rng(seed)
    pick = {0, nb - 1}
    pick.update(int(x) for x in rng.choice(np.arange(1, nb - 1), size=min(n_random, nb - 2), replace=False))
    return sorted(pick)


# Per-case parity summaries of this pytest session (printed at its end by
# the terminal-summary hook in conftest.py): how many routing decisions and
# blocks fell in the 1e-4 exemption band (exempt_routes, exempt_blocks), how
# many of those the GPU actually decided differently from the oracle
# (routes_differing, exempt_differing; every decision outside the band is
# equal, or the test fails), and the attention errors.
SESSION_REPORTS = []


def record(case: str, reps, **extra) -> dict:
    """Adds one parity case's summary to SESSION_REPORTS and returns it."""
    rec = {"case": case, "heads": len(reps),
           "vs_heads": sum(1 for r in reps if r.get("pattern") == O.VS),
           "exempt_routes": sum(int(r["exempt_route"]) for r in reps),
           "exempt_blocks": sum(int(r["exempt_blocks"]) for r in reps),
           "exempt_differing": sum(int(r["exempt_differing"]) for r in reps),
           "routes_differing": sum(int(r["route_differs"]) for r in reps),
           "qblocks_compared": sum(int(r.get("qblocks", 0)) for r in reps),
           "attn_max_abs": max((r["attn_max_abs"] for r in reps), default=0.0),
           "attn_mean_abs": max((r["attn_mean_abs"] for r in reps), default=0.0),
           "density": (sum(r["density"] for r in reps) / len(reps)) if reps else 0.0}
    rec.update(extra)
    SESSION_REPORTS.append(rec)
    return rec


def compare_all(w, q, k, v, gpu, oprm, qblocks_fn=None, heads=None):
    g = w.h_q // w.h_kv
    reports = []
    for b in range(w.batch):
        for h in (range(w.h_q) if heads is None else heads):
            n = w.length(b)
            qh = O.bf16_to_f64(q[b, h, :n])
            kh = O.bf16_to_f64(k[b, h // g, :n])
            vh = O.bf16_to_f64(v[b, h // g, :n])
            qbs = None if qblocks_fn is None else qblocks_fn(b, h)
            reports.append(compare_head(gpu, b, h, qh, kh, vh, w, oprm, qbs))
    return reports
