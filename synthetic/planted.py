"""Planted-structure Q/K/V generator (bf16, layout [batch, heads, seq, dim]).

Recipe (every amplitude is in logit units: a component ``a`` placed in Q and
``b`` in K along the same coordinate direction, each scaled by ``dim**0.25``,
adds exactly ``a*b`` to the scaled logit ``q.k/sqrt(dim)``):

* base: Q, K, V entries ~ N(0,1)/sqrt(dim). K's base noise is left out of the
  18 planted coordinate directions (dims 0..17) so that the block-level
  background stays flat, as in the two-level signal/background model of the
  CRISP paper's Appendix C.
* sink: K rows 0..3 get +4 along e16; Q rows of vertical-slash (VS) heads get
  +c along e16, i.e. a sink logit of 4c.
* verticals: ``n_vertical`` key rows per KV head, uniform in [block, N-block),
  get +3 along e17; VS query heads get +2 along e17 (logit +6).
* recency: 8 RoPE-style (cos, sin) pairs in dims 0..15, on Q of VS heads and
  on all of K, with peak logit ``recency_peak`` at zero offset.
  ``recency_freqs="rope"`` uses the usual geometric frequencies
  10000**(-k/8); ``"block"`` uses frequencies 2*pi*(k+1)/block, whose
  block sums are the same for every key block (no far-field structure).
* diffuse heads: Q carries no planted component (near-uniform causal head).
* variable lengths: with ``lengths`` set, batch element b is a sequence of
  lengths[b] tokens stored in the first lengths[b] rows of its [seqlen, d]
  slices (verticals drawn inside it); the remaining rows are padding,
  filled with large finite values (N(0,1) * 64) that the method must ignore.

Seeds: every (tensor, batch, head) slice has its own generator seeded from
``numpy.random.SeedSequence``; planted positions and per-head amplitudes
come from ``numpy.random.default_rng(seed)``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

SINK_DIM = 16
VERT_DIM = 17
N_RESERVED = 18
N_SINK_ROWS = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention workload (shapes + planted structure)."""

    name: str
    batch: int
    h_q: int
    h_kv: int
    head_dim: int
    seqlen: int
    block: int
    diffuse_frac: float = 0.25
    diffuse_heads: Optional[Sequence[int]] = None  # explicit list overrides diffuse_frac
    sink_logit: float = 12.0                        # logit of a sink key for VS heads
    sink_logit_range: Optional[Sequence[float]] = None  # (lo, hi): per-head U[lo,hi]*3
    n_vertical: int = 8
    recency_peak: float = 3.0
    recency_freqs: str = "block"
    v_unit: bool = False      # V ~ N(0,1) instead of N(0,1)/sqrt(dim)
    seed: int = 0
    lengths: Optional[Sequence[int]] = None   # per-batch sequence lengths (<= seqlen)

    @property
    def n_blocks(self) -> int:
        """Blocks of the longest sequence, ceil(seqlen / block)."""
        return -(-self.seqlen // self.block)

    def length(self, b: int) -> int:
        return self.seqlen if self.lengths is None else int(self.lengths[b])

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# Llama-3.1-8B / Qwen2.5-7B single-layer attention shapes.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 1, 64, 2048, 64, diffuse_heads=(1,), sink_logit=8.0,
                     n_vertical=0, recency_peak=9.0, recency_freqs="rope"),
    "llama_32k": Workload("llama_32k", 1, 32, 8, 128, 32768, 128),
    "qwen_131k": Workload("qwen_131k", 1, 28, 4, 128, 131072, 128, sink_logit_range=(1.0, 6.0)),
    "llama_8k": Workload("llama_8k", 1, 32, 8, 128, 8192, 128),
    "llama_128k": Workload("llama_128k", 1, 32, 8, 128, 131072, 128),
    "llama_512k": Workload("llama_512k", 1, 32, 8, 128, 524288, 128),
    # the same shapes with a decaying RoPE-style recency band (geometric
    # frequencies 10000**(-k/8), peak logit 9) instead of the block-periodic one
    "llama_32k_rope": Workload("llama_32k_rope", 1, 32, 8, 128, 32768, 128, recency_peak=9.0,
                               recency_freqs="rope"),
    "llama_512k_rope": Workload("llama_512k_rope", 1, 32, 8, 128, 524288, 128, recency_peak=9.0,
                                recency_freqs="rope"),
    # four prompts of different lengths (none a multiple of the block but the
    # first) in one padded batch
    "llama_varlen_131k": Workload("llama_varlen_131k", 4, 32, 8, 128, 131072, 128,
                                  lengths=(131072, 98304 + 37, 65536 + 1, 32768 + 123)),
}


def sweep_workload(seqlen: int, diffuse_frac: float) -> Workload:
    """Llama-shaped sweep point (seq length x diffuse-head fraction)."""
    return Workload(f"llama_{seqlen // 1024}k_f{diffuse_frac:g}", 1, 32, 8, 128, seqlen, 128,
                    diffuse_frac=diffuse_frac)


def _slice_seed(seed: int, *tags: int) -> int:
    ss = np.random.SeedSequence([seed, *tags])
    return int(ss.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1))


def head_kinds(w: Workload) -> Dict[str, object]:
    """Planted layout: which query heads are diffuse, sink logits, vertical rows."""
    rng = np.random.default_rng(w.seed)
    if w.diffuse_heads is not None:
        diffuse = sorted(int(h) for h in w.diffuse_heads)
    else:
        perm = rng.permutation(w.h_q)
        diffuse = sorted(int(h) for h in perm[: int(round(w.diffuse_frac * w.h_q))])
    if w.sink_logit_range is not None:
        lo, hi = w.sink_logit_range
        sink = (3.0 * rng.uniform(lo, hi, size=w.h_q)).tolist()
    else:
        sink = [float(w.sink_logit)] * w.h_q
    verticals: List[List[int]] = []
    for i in range(w.batch * w.h_kv):
        if w.n_vertical:
            n_b = w.length(i // w.h_kv)
            verticals.append(sorted(int(x) for x in rng.integers(w.block, n_b - w.block,
                                                                   size=w.n_vertical)))
        else:
            verticals.append([])
    return {"diffuse": diffuse, "sink_logit": sink, "verticals": verticals}


def _recency_omega(w: Workload) -> np.ndarray:
    k = np.arange(8, dtype=np.float64)
    if w.recency_freqs == "rope":
        return 10000.0 ** (-k / 8.0)
    if w.recency_freqs == "block":
        return 2.0 * math.pi * (k + 1.0) / w.block
    raise ValueError(w.recency_freqs)


def _rope_block(w: Workload, pos: torch.Tensor, amp: float) -> torch.Tensor:
    om = torch.tensor(_recency_omega(w), dtype=torch.float64, device=pos.device)
    ang = pos.to(torch.float64)[:, None] * om[None, :]
    out = torch.empty(pos.numel(), 16, dtype=torch.float64, device=pos.device)
    out[:, 0::2] = amp * torch.cos(ang)
    out[:, 1::2] = amp * torch.sin(ang)
    return out.to(torch.float32)


def make_qkv(w: Workload, device: str = "cpu", heads_q: Optional[Sequence[int]] = None,
             heads_kv: Optional[Sequence[int]] = None):
    """Return (q, k, v, meta) as bf16 tensors [B, H, N, d] on ``device``.

    ``heads_q`` restricts generation to a subset of query heads (their KV
    heads are generated in full); the returned q then holds only those heads.
    ``heads_kv`` restricts k and v to those KV heads and, unless heads_q is
    given, q to their query heads: a slice of the whole problem, with the
    same values the whole generation gives those heads (every slice has its
    own seeded generator).
    """
    d, N = w.head_dim, w.seqlen
    c4 = d ** 0.25
    meta = head_kinds(w)
    diffuse = set(meta["diffuse"])
    g = w.h_q // w.h_kv
    hk_list = list(range(w.h_kv)) if heads_kv is None else list(heads_kv)
    if heads_q is not None:
        hq_list = list(heads_q)
    else:
        hq_list = [hk * g + i for hk in hk_list for i in range(g)]
    rec_amp = math.sqrt(w.recency_peak / 8.0) * c4
    pos = torch.arange(N, device=device)
    rope = _rope_block(w, pos, rec_amp) if w.recency_peak > 0 else None

    def randn(tag: int, b: int, h: int) -> torch.Tensor:
        gen = torch.Generator(device=device)
        gen.manual_seed(_slice_seed(w.seed, tag, b, h))
        return torch.randn((N, d), generator=gen, device=device, dtype=torch.float32)

    inv = 1.0 / math.sqrt(d)
    q = torch.empty((w.batch, len(hq_list), N, d), dtype=torch.bfloat16, device=device)
    k = torch.empty((w.batch, len(hk_list), N, d), dtype=torch.bfloat16, device=device)
    v = torch.empty((w.batch, len(hk_list), N, d), dtype=torch.bfloat16, device=device)

    def pad(x: torch.Tensor, tag: int, b: int, h: int) -> torch.Tensor:
        n_b = w.length(b)
        if n_b < N:
            gen = torch.Generator(device=device)
            gen.manual_seed(_slice_seed(w.seed, tag, b, h))
            x[n_b:] = torch.randn((N - n_b, d), generator=gen, device=device, dtype=torch.float32) * 64.0
        return x
    for b in range(w.batch):
        for j, hk in enumerate(hk_list):
            x = randn(1, b, hk).mul_(inv)
            x[:, :N_RESERVED] = 0.0
            x[:N_SINK_ROWS, SINK_DIM] += 4.0 * c4
            for p in meta["verticals"][b * w.h_kv + hk]:
                x[p, VERT_DIM] += 3.0 * c4
            if rope is not None:
                x[:, :16] += rope
            k[b, j] = pad(x, 11, b, hk).to(torch.bfloat16)
            x = randn(2, b, hk)
            if not w.v_unit:
                x.mul_(inv)
            v[b, j] = pad(x, 12, b, hk).to(torch.bfloat16)
        for i, h in enumerate(hq_list):
            x = randn(0, b, h).mul_(inv)
            if h not in diffuse:
                x[:, SINK_DIM] += (meta["sink_logit"][h] / 4.0) * c4
                if w.n_vertical:
                    x[:, VERT_DIM] += 2.0 * c4
                if rope is not None:
                    x[:, :16] += rope
            q[b, i] = pad(x, 10, b, h).to(torch.bfloat16)
    meta = dict(meta)
    meta["group"] = g
    return q, k, v, meta
