"""Algorithmic FLOP and byte counts for attention decode, as the "MLA Cost
Analysis & Regime Guide" page states them (section "Cost Models",
DeepSeek-V3-like h=128, d=128, k=512, p=64; w = bytes per element).

* FlashMLA / latent space:  FLOPs = 2 b h s t (2k + p)
                            bytes = w (b h s (2k + p) + b t (k + p))
* FlashAttention, decompressed: FLOPs = 2 b h s t (2d + p)
                                bytes = w b h (s + t) (2d + p)
* MLAvar6+ split cache (o latent tokens + n decompressed, t = o + n):
      FLOPs = 2bhstp + 4bhsnd + 4bhsok
      bytes = w (bhsp + bhsd + bhsk + bok + btp + 2 bhnd + bhsd + bhsk)

For a jagged batch the per-request context lengths are summed: b*t becomes
sum_r t_r.  The causal saving among s speculative tokens is ignored, as the
page's model ignores it.  For an FP8 latent cache each cached token costs
512 e4m3 bytes + one fp32 scale + 64 bf16 RoPE values.
"""
from __future__ import annotations

H, D, K, P = 128, 128, 512, 64


def mla_flops(b, h, s, t, k=K, p=P, sum_t=None):
    bt = b * t if sum_t is None else sum_t
    return 2.0 * h * s * bt * (2 * k + p)


def mla_bytes(b, h, s, t, k=K, p=P, w=2, sum_t=None, cache_bytes_per_token=None):
    bt = b * t if sum_t is None else sum_t
    io = w * b * h * s * (2 * k + p)
    cache = w * bt * (k + p) if cache_bytes_per_token is None else bt * cache_bytes_per_token
    return float(io + cache)


def fa_flops(b, h, s, t, d=D, p=P):
    return 2.0 * b * h * s * t * (2 * d + p)


def fa_bytes(b, h, s, t, d=D, p=P, w=2):
    return float(w * b * h * (s + t) * (2 * d + p))


def mlavar6_flops(b, h, s, o, n, d=D, k=K, p=P):
    t = o + n
    return 2.0 * b * h * s * t * p + 4.0 * b * h * s * n * d + 4.0 * b * h * s * o * k


def mlavar6_bytes(b, h, s, o, n, d=D, k=K, p=P, w=2):
    t = o + n
    return float(w * (b * h * s * p + b * h * s * d + b * h * s * k + b * o * k + b * t * p
                      + 2 * b * h * n * d + b * h * s * d + b * h * s * k))


FP8_CACHE_BYTES_PER_TOKEN = K + 4 + 2 * P   # e4m3 latent + fp32 scale + bf16 RoPE


def workload_cost(wl):
    """(FLOPs, bytes) of one decode step over a Workload from mla_workloads."""
    st = wl.total_tokens
    flops = mla_flops(wl.batch, wl.num_heads, wl.s_q, None, sum_t=st)
    cb = FP8_CACHE_BYTES_PER_TOKEN if wl.cache_dtype == "fp8" else None
    nbytes = mla_bytes(wl.batch, wl.num_heads, wl.s_q, None, sum_t=st, cache_bytes_per_token=cb)
    return flops, nbytes
