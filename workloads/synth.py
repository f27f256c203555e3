"""Seeded synthetic inputs for hierarchical top-p sparse decode attention.

This module only draws random numbers and lays them out the way a paged KV cache is laid out.
It holds none of the method's arithmetic (no bounds, no quantisation, no scoring, no top-p, no
attention), so the CUDA path and the CPU oracle can both be fed from it without sharing any
computation.

Workload recipes follow the decode settings of "Twilight: Adaptive Attention Sparsity with
Hierarchical Top-p Pruning" (paperlayer summary, section 5.2 and appendix B.2: GQA decode over a
paged fp16 KV cache with 16-token pages; notes page, "Key findings": per-head budgets differ up to
50x).  The pages evaluate on LongBench / RULER with LLaMA-family weights, which are not available;
these generators stand in with the structure those heads show: a few heavy tokens, attention sinks
at positions 0-3, and per-head temperatures that mix focused and diffuse heads.

Layouts (all numpy, C-contiguous):
  q           fp16  [B][Hq][D]
  k, v        fp16  [P_phys][Hkv][page_size][D]
  page_table  int32 [B][max_pages]   logical page -> physical page, -1 past the sequence
  seq_lens    int32 [B]
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

HEAD_DIM = 128
PAGE_SIZE = 16


@dataclass
class DecodeWorkload:
    name: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    page_table: np.ndarray
    seq_lens: np.ndarray
    num_q_heads: int
    num_kv_heads: int
    p: float = 0.85
    eps: float = 1e-6
    budget_div: int = 4
    budget_pages: int = 0
    head_dim: int = HEAD_DIM
    page_size: int = PAGE_SIZE
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.q.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def num_phys_pages(self) -> int:
        return int(self.k.shape[0])


def _pages(n: int) -> int:
    return (n + PAGE_SIZE - 1) // PAGE_SIZE


def _unit(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x)


def make_decode(name: str, batch: int, num_q_heads: int, num_kv_heads: int, seq_lens,
                seed: int = 0, tau=None, tau_range=(0.25, 8.0), heavy_frac: float = 0.01,
                heavy_count: int | None = None, num_sinks: int = 4, heavy_coef: float = 3.0,
                sink_coef: float = 2.0, spans: int = 0, span_len: int = 512,
                permute_pages: bool = False, max_pages: int | None = None,
                p: float = 0.85, eps: float = 1e-6, budget_div: int = 4,
                budget_pages: int = 0, temperature: bool = False) -> DecodeWorkload:
    """Draw one decode layer.

    K, V ~ N(0, 1) per channel.  Query q_h = tau_h * g_h with g_h ~ N(0, I_D), or, with
    ``temperature``, q_h = g_h / tau_h (tau_h is then a logit temperature: every logit of head h
    is divided by it); tau_h is fixed (``tau``) or log-uniform in ``tau_range``.  Per (b, kv-head): ``heavy_count`` (default
    round(heavy_frac * N_b)) heavy tokens, each aimed at one q-head h* of the group,
    K_i = heavy_coef * sqrt(D) * q_h*/|q_h*| + xi; positions uniform in [num_sinks, N_b) or, with
    ``spans`` > 0, uniform inside that head's spans of ``span_len`` tokens.  Sink tokens 0..3:
    K_i = sink_coef * sqrt(D) * u + xi with u the normalised mean of the group's unit queries.
    """
    rng = np.random.default_rng(seed)
    d = HEAD_DIM
    g = num_q_heads // num_kv_heads
    assert num_q_heads % num_kv_heads == 0
    seq_lens = np.asarray(seq_lens, dtype=np.int64).reshape(batch)
    n_pages = np.array([_pages(int(n)) for n in seq_lens], dtype=np.int64)
    if max_pages is None:
        max_pages = int(n_pages.max())
    p_phys = int(n_pages.sum())

    # page table: identity blocks, or one random permutation dealt to sequences in order
    page_table = np.full((batch, max_pages), -1, dtype=np.int32)
    phys_ids = rng.permutation(p_phys) if permute_pages else np.arange(p_phys)
    off = 0
    for b in range(batch):
        page_table[b, : n_pages[b]] = phys_ids[off: off + n_pages[b]]
        off += int(n_pages[b])

    # queries
    gq = rng.standard_normal((batch, num_q_heads, d))
    if tau is None:
        lo, hi = np.log(tau_range[0]), np.log(tau_range[1])
        taus = np.exp(rng.uniform(lo, hi, size=(batch, num_q_heads)))
    else:
        taus = np.full((batch, num_q_heads), float(tau))
    q64 = gq / taus[:, :, None] if temperature else gq * taus[:, :, None]
    q = q64.astype(np.float16)

    # base K, V in physical layout (bulk normals from a seeded torch CPU generator: faster
    # than numpy's for hundreds of millions of draws)
    tg = torch.Generator().manual_seed(int(seed))
    k = torch.randn((p_phys, num_kv_heads, PAGE_SIZE, d), generator=tg,
                    dtype=torch.float32).numpy()
    v = torch.randn((p_phys, num_kv_heads, PAGE_SIZE, d), generator=tg,
                    dtype=torch.float16)

    def locate(b: int, pos: int):
        return int(page_table[b, pos // PAGE_SIZE]), pos % PAGE_SIZE

    sqrt_d = np.sqrt(d)
    heavy_log = []
    for b in range(batch):
        nb = int(seq_lens[b])
        for kvh in range(num_kv_heads):
            heads = list(range(kvh * g, (kvh + 1) * g))
            units = [_unit(q64[b, h]) for h in heads]
            # sinks
            u = _unit(np.mean(units, axis=0))
            for pos in range(min(num_sinks, nb)):
                ph, r = locate(b, pos)
                k[ph, kvh, r] += sink_coef * sqrt_d * u
            # heavy tokens
            cnt = heavy_count if heavy_count is not None else int(round(heavy_frac * nb))
            lo_pos = min(num_sinks, nb)
            if cnt <= 0 or nb - lo_pos <= 0:
                continue
            owners = rng.integers(0, g, size=cnt)
            if spans > 0:
                starts = rng.integers(lo_pos, max(lo_pos + 1, nb - span_len + 1),
                                      size=(g, spans))
                which = rng.integers(0, spans, size=cnt)
                offs = rng.integers(0, span_len, size=cnt)
                pos_all = np.minimum(starts[owners, which] + offs, nb - 1)
            else:
                cnt = min(cnt, nb - lo_pos)
                pos_all = lo_pos + rng.choice(nb - lo_pos, size=cnt, replace=False)
                owners = owners[:cnt]
            noise = rng.standard_normal((len(pos_all), d))
            uvec = np.stack(units)[owners]
            phys = page_table[b, pos_all // PAGE_SIZE]
            # assignment (not accumulation): a repeated position stays one heavy token
            k[phys, kvh, pos_all % PAGE_SIZE] = (heavy_coef * sqrt_d * uvec
                                                 + noise).astype(np.float32)
            heavy_log.extend((b, kvh, int(pp), heads[o])
                             for pp, o in zip(pos_all.tolist(), owners.tolist()))

    wl = DecodeWorkload(
        name=name, q=q, k=torch.from_numpy(k).half().numpy(), v=v.numpy(),
        page_table=page_table, seq_lens=seq_lens.astype(np.int32),
        num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, p=p, eps=eps,
        budget_div=budget_div, budget_pages=budget_pages,
        extra={"tau": taus, "heavy": heavy_log, "seed": seed})
    return wl


# ---------------------------------------------------------------------------------------------
# The five workload shapes (full size) and reduced variants with the same recipe.
# ---------------------------------------------------------------------------------------------

def config1(seed: int = 0, n: int = 4096) -> DecodeWorkload:
    """Single-head decode, batch 1, 4096 tokens, tau = 2, 16 heavy tokens, 4 sinks."""
    return make_decode("c1_single_head_4k", 1, 1, 1, [n], seed=seed, tau=2.0,
                       heavy_count=16 * n // 4096)


def config2(seed: int = 0, n: int = 32768, batch: int = 1) -> DecodeWorkload:
    """Llama-3.1-8B-shaped GQA layer (32 q-heads / 8 kv-heads), batch 1, 32K context; per-head
    logit temperature log-uniform in [0.25, 8] (focused and diffuse heads)."""
    return make_decode(f"c2_gqa_b{batch}_{n // 1024}k", batch, 32, 8, [n] * batch, seed=seed,
                       temperature=True)


def config3(seed: int = 0, batch: int = 16, n_lo: int = 8192, n_hi: int = 32768,
            num_q_heads: int = 32, num_kv_heads: int = 8) -> DecodeWorkload:
    """Batch 16, per-sequence lengths uniform in [8192, 32768], pages randomly permuted."""
    rng = np.random.default_rng(seed + 1_000_003)
    lens = rng.integers(n_lo, n_hi + 1, size=batch)
    max_pages = _pages(n_hi)
    return make_decode(f"c3_gqa_b{batch}_{n_lo // 1024}k-{n_hi // 1024}k", batch, num_q_heads,
                       num_kv_heads, lens, seed=seed, permute_pages=True, max_pages=max_pages,
                       temperature=True)


def config4(seed: int = 0, n: int = 131072, batch: int = 4, p: float = 0.85) -> DecodeWorkload:
    """Long context, batch 4, heavy tokens clustered in 8 spans of 512 tokens per head."""
    return make_decode(f"c4_gqa_b{batch}_{n // 1024}k_p{int(round(p * 100))}", batch, 32, 8,
                       [n] * batch, seed=seed, spans=8, span_len=min(512, max(16, n // 16)),
                       p=p, temperature=True)


def config6(seed: int = 0, batch: int = 64, n: int = 8192) -> DecodeWorkload:
    """Serving batch: 64 sequences of 8192 tokens, 32/8 heads, pages randomly permuted."""
    return make_decode(f"c6_gqa_b{batch}_{n // 1024}k", batch, 32, 8, [n] * batch, seed=seed,
                       permute_pages=True, temperature=True)


def config_diffuse(seed: int = 0, n: int = 32768, batch: int = 1) -> DecodeWorkload:
    """The 32K GQA layer with diffuse heads only: no heavy tokens (sinks kept), logit temperature
    log-uniform in [2, 8], so every head spreads its weight over most of its candidates."""
    return make_decode(f"c2_diffuse_b{batch}_{n // 1024}k", batch, 32, 8, [n] * batch,
                       seed=seed, temperature=True, heavy_frac=0.0, tau_range=(2.0, 8.0))


def config5_rows(rows: int, n: int, seed: int = 0, tie_frac: float = 0.01):
    """Standalone pruner input: ``rows`` probability vectors of length n (fp32).

    Half the rows are Gaussian-logit rows (sigma log-uniform in [0.1, 6]), half are Zipf rank
    profiles w_r ~ r^-s (s ~ U[0.5, 2]) with ranks permuted over positions.  A ``tie_frac`` share
    of rows carries exact ties: Gaussian logits rounded to multiples of 1/8, Zipf ranks merged in
    groups of four.  Each row is normalised to sum to one in fp64, then rounded to fp32.
    Returns (w fp32 [rows][n], info dict).
    """
    rng = np.random.default_rng(seed)
    w = np.empty((rows, n), dtype=np.float32)
    fam = rng.integers(0, 2, size=rows)
    n_tie = max(1, int(round(tie_frac * rows))) if tie_frac > 0 else 0
    ties = np.zeros(rows, dtype=bool)
    ties[rng.choice(rows, size=n_tie, replace=False)] = True
    params = np.empty(rows)
    for r in range(rows):
        if fam[r] == 0:
            sigma = float(np.exp(rng.uniform(np.log(0.1), np.log(6.0))))
            logit = rng.standard_normal(n) * sigma
            if ties[r]:
                logit = np.round(logit * 8.0) / 8.0
            e = np.exp(logit - logit.max())
            params[r] = sigma
        else:
            s = float(rng.uniform(0.5, 2.0))
            rank = np.arange(1, n + 1, dtype=np.float64)
            if ties[r]:
                rank = np.ceil(rank / 4.0)
            e = rank ** (-s)
            e = e[rng.permutation(n)]
            params[r] = s
        w[r] = (e / e.sum()).astype(np.float32)
    return w, {"family": fam, "ties": ties, "param": params, "seed": seed}


CONFIG_NAMES = {
    1: "single-head decode, B=1, 1/1 heads, 4096 ctx",
    2: "GQA decode layer, B=1, 32/8 heads, 32768 ctx",
    3: "GQA decode layer, B=16, 32/8 heads, ctx U[8192,32768], permuted pages",
    4: "GQA decode layer, B=4, 32/8 heads, 131072 ctx, clustered heavy spans",
    5: "standalone top-p pruner, 4096 rows x n in {8192, 32768, 131072}",
}
