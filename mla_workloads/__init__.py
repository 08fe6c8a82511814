"""Seeded synthetic inputs for MLA decode in absorbed latent space.

This module only *draws* inputs: the absorbed query rows, the paged latent+RoPE
cache, the block table and the sequence lengths.  It holds none of the
attention arithmetic, so both the CUDA path and the fp64 oracle can consume
what it produces without sharing any computation.

Shapes follow the DeepSeek-V3 defaults of the "MLA Cost Analysis & Regime
Guide" page (section "Tensor Shapes"): h=128 heads, latent k=512, RoPE p=64,
so one cache row is 576 values and the value rows are its first 512.

Recipe (every workload; all draws from one ``torch.Generator`` seeded per
workload, in this order):

1. sequence lengths (only the jagged workload draws them),
2. a random permutation of the page pool (the block table),
3. the query tensor Q, shape (b, s_q, h, 576), N(0, 1) rounded to bf16,
4. the cache rows, N(0, 1) rounded to bf16, page by page in pool order.

The FP8 workload quantises the bf16 latent part of each cache row with one
fp32 scale per token (scale = amax / 448, amax over the 512 latent values,
round-to-nearest-even to e4m3 with saturation at +-448; amax = 0 gives scale
1).  The RoPE part stays bf16.  That quantisation is data preparation: the
kernel and the oracle both read the same stored bytes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

PAGE = 64            # tokens per KV page
D_QK = 576           # k + p: latent 512 + RoPE 64
D_V = 512            # k: value rows are the first 512 values of a cache row
D_ROPE = D_QK - D_V
FP8_PAGE_BYTES = PAGE * D_V + PAGE * D_ROPE * 2   # e4m3 plane + bf16 RoPE plane
FP8_MAX = 448.0
DEFAULT_SCALE = 1.0 / math.sqrt(192.0)           # 1/sqrt(d + p), d=128, p=64


@dataclasses.dataclass
class Workload:
    """One decode batch held in host memory (CPU tensors / numpy arrays)."""

    name: str
    batch: int
    s_q: int
    num_heads: int
    causal: bool
    cache_dtype: str                  # "bf16" or "fp8"
    seqlens: np.ndarray               # int32 [b]
    block_table: np.ndarray           # int32 [b, max_pages]
    q: torch.Tensor                   # bf16 [b, s_q, h, 576]
    pool: torch.Tensor                # bf16 [P, 64, 576]  or uint8 [P, FP8_PAGE_BYTES]
    kv_scale: Optional[torch.Tensor]  # fp32 [P, 64] for fp8, else None
    softmax_scale: float = DEFAULT_SCALE
    seed: int = 0

    @property
    def num_pages(self) -> int:
        return int(self.pool.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def total_tokens(self) -> int:
        return int(self.seqlens.astype(np.int64).sum())

    def describe(self) -> dict:
        return {"workload": self.name, "batch": self.batch, "s_q": self.s_q,
                "heads": self.num_heads, "d_qk": D_QK, "d_v": D_V, "page": PAGE,
                "sum_t": self.total_tokens, "cache": self.cache_dtype,
                "causal": self.causal, "seed": self.seed}


def jagged_lengths(gen: torch.Generator, batch: int, lo: int = 128, hi: int = 131072) -> np.ndarray:
    """batch-2 lengths round(exp(U[ln lo, ln hi])) plus one forced lo and one
    forced hi, shuffled with the same generator."""
    u = torch.rand(batch - 2, generator=gen, dtype=torch.float64)
    lens = torch.round(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    lens = torch.cat([lens, torch.tensor([float(lo), float(hi)], dtype=torch.float64)])
    perm = torch.randperm(batch, generator=gen)
    return lens[perm].to(torch.int64).numpy().astype(np.int32)


def _block_table(gen: torch.Generator, seqlens: np.ndarray, contiguous: bool):
    pages = [(int(t) + PAGE - 1) // PAGE for t in seqlens]
    total = sum(pages)
    max_pages = max(1, max(pages) if pages else 1)
    if contiguous:
        order = torch.arange(total, dtype=torch.int64)
    else:
        order = torch.randperm(total, generator=gen)
    table = np.zeros((len(seqlens), max_pages), dtype=np.int32)
    off = 0
    for r, n in enumerate(pages):
        table[r, :n] = order[off:off + n].numpy()
        off += n
    return table, total


def _randn_bf16(gen: torch.Generator, shape, chunk_rows: int = 4096) -> torch.Tensor:
    """N(0,1) rounded to bf16, drawn in row chunks so that huge pools never
    materialise as fp32 all at once."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(shape[0], -1)
    for i in range(0, shape[0], chunk_rows):
        j = min(shape[0], i + chunk_rows)
        flat[i:j] = torch.randn((j - i, flat.shape[1]), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return out


def quantize_fp8_pages(src: torch.Tensor):
    """bf16 pages [P, 64, 576] -> (uint8 pages [P, FP8_PAGE_BYTES], fp32 scales [P, 64]).

    Byte layout of one page: 64x512 e4m3 latent values (token-major), then
    64x64 bf16 RoPE values (token-major)."""
    P = src.shape[0]
    lat = src[:, :, :D_V].to(torch.float32)
    amax = lat.abs().amax(dim=2)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax)).to(torch.float32)
    qv = (lat / scale[:, :, None]).clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    out = torch.empty((P, FP8_PAGE_BYTES), dtype=torch.uint8)
    out[:, :PAGE * D_V] = qv.view(torch.uint8).reshape(P, PAGE * D_V)
    rope = src[:, :, D_V:].contiguous().view(torch.uint8).reshape(P, PAGE * D_ROPE * 2)
    out[:, PAGE * D_V:] = rope
    return out, scale


def make(batch: int, s_q: int, num_heads: int, seqlens, *, causal: bool = False,
         cache_dtype: str = "bf16", contiguous: bool = False, seed: int = 0,
         name: str = "custom", jagged: Optional[tuple] = None,
         softmax_scale: float = DEFAULT_SCALE) -> Workload:
    """Generic generator.  ``seqlens`` is an int or a sequence; with
    ``jagged=(lo, hi)`` the lengths are drawn instead (``seqlens`` ignored)."""
    gen = torch.Generator().manual_seed(seed)
    if jagged is not None:
        lens = jagged_lengths(gen, batch, *jagged)
    elif np.isscalar(seqlens):
        lens = np.full(batch, int(seqlens), dtype=np.int32)
    else:
        lens = np.asarray(seqlens, dtype=np.int32)
        assert lens.shape == (batch,)
    table, total_pages = _block_table(gen, lens, contiguous)
    q = _randn_bf16(gen, (batch, s_q, num_heads, D_QK))
    src = _randn_bf16(gen, (max(total_pages, 1), PAGE, D_QK))
    kv_scale = None
    pool = src
    if cache_dtype == "fp8":
        pool, kv_scale = quantize_fp8_pages(src)
    elif cache_dtype != "bf16":
        raise ValueError(cache_dtype)
    return Workload(name=name, batch=batch, s_q=s_q, num_heads=num_heads, causal=causal,
                    cache_dtype=cache_dtype, seqlens=lens, block_table=table, q=q,
                    pool=pool, kv_scale=kv_scale, softmax_scale=softmax_scale, seed=seed)


# The five decode workloads.  Config 2 is the headline one (b=64, h=128,
# t=4096: the shape the page's cost-model arithmetic intensity is quoted on).
CONFIGS = {
    1: dict(name="tiny_b2_h16_t256_contig", batch=2, s_q=1, num_heads=16, seqlens=256, contiguous=True),
    2: dict(name="dsv3_b64_h128_t4096_paged", batch=64, s_q=1, num_heads=128, seqlens=4096),
    3: dict(name="jagged_b128_h128_t128-131072", batch=128, s_q=1, num_heads=128, seqlens=None,
            jagged=(128, 131072)),
    4: dict(name="fp8_b64_h128_t32768", batch=64, s_q=1, num_heads=128, seqlens=32768, cache_dtype="fp8"),
    5: dict(name="spec_b32_s16_h128_t4096_causal", batch=32, s_q=16, num_heads=128, seqlens=4096, causal=True),
}


def make_config(cfg: int, seed: int = 0) -> Workload:
    kw = dict(CONFIGS[cfg])
    return make(seed=seed, **kw)


def config_shape(cfg: int, seed: int = 0):
    """(batch, s_q, heads, seqlens) without drawing the tensors."""
    kw = dict(CONFIGS[cfg])
    if kw.get("jagged"):
        lens = jagged_lengths(torch.Generator().manual_seed(seed), kw["batch"], *kw["jagged"])
    else:
        lens = np.full(kw["batch"], kw["seqlens"], dtype=np.int32)
    return kw["batch"], kw["s_q"], kw["num_heads"], lens


D_HEAD = 128         # d: per-head query / key / value dims before absorption


@dataclasses.dataclass
class Projections:
    """Inputs of the two per-head projections around the latent attention.

    q       bf16 [rows, h, d + p]: [q_nope | q_pe] per head
    w_k     bf16 [h, 512, d]: head j's keys are K_j = Z . w_k[j]
    o_lat   bf16 [rows, h, 512]: latent attention output rows
    w_kvb2  bf16 [h, d, 512]: head j's values are V_j = Z . w_kvb2[j]^T
    """
    q: torch.Tensor
    w_k: torch.Tensor
    o_lat: torch.Tensor
    w_kvb2: torch.Tensor


def make_projections(rows: int, num_heads: int, seed: int = 0) -> Projections:
    """Draws, in this order from one generator: q ~ N(0, 1); w_k ~
    N(0, 1/d) (so the absorbed latent query is about unit variance);
    o_lat ~ N(0, 1); w_kvb2 ~ N(0, 1/512).  Every draw is rounded to bf16."""
    gen = torch.Generator().manual_seed(seed)
    h = num_heads
    q = _randn_bf16(gen, (rows, h, D_HEAD + D_ROPE)) if rows else torch.empty((0, h, D_HEAD + D_ROPE),
                                                                               dtype=torch.bfloat16)
    w_k = (torch.randn((h, D_V, D_HEAD), generator=gen) / math.sqrt(D_HEAD)).to(torch.bfloat16)
    o_lat = _randn_bf16(gen, (rows, h, D_V)) if rows else torch.empty((0, h, D_V), dtype=torch.bfloat16)
    w_kvb2 = (torch.randn((h, D_HEAD, D_V), generator=gen) / math.sqrt(D_V)).to(torch.bfloat16)
    return Projections(q, w_k, o_lat, w_kvb2)


def make_sparse_indices(seqlens, s_q: int, topk: int, seed: int = 0, pad: int = 0) -> np.ndarray:
    """Per query token, `topk - pad` distinct cache positions drawn uniformly
    from the request's [0, t) (all of them, in random order, when t is
    smaller), then -1 up to `topk`: int32 [b, s_q, topk].  Draws from one
    generator, request by request, query token by query token."""
    gen = torch.Generator().manual_seed(seed)
    b = len(seqlens)
    out = np.full((b, s_q, topk), -1, dtype=np.int32)
    for r in range(b):
        t = int(seqlens[r])
        for i in range(s_q):
            n = min(topk - pad, t)
            if n > 0:
                out[r, i, :n] = torch.randperm(t, generator=gen)[:n].numpy()
    return out
