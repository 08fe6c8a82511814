"""GPU parity of the MLAvar6+ split decode (mla_var6_decode_fwd through the C
ABI) against the fp64 oracle of the split form, oracle.mlavar6_decode, at the
decode contract's bars: O max |err| <= 2e-2, relative L1 against the
bf16-rounded oracle <= 1e-3, lse max |err| <= 1e-3.  The library carries its
two intermediates (the latent output of the old tokens and its
decompression) as two bf16 terms each, so the split path adds no rounding of
its own to the decode's.
"""
import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
import mla_workloads as mw
import oracle
from gpu_helpers import LSE_MAX_ABS, O_MAX_ABS, O_REL_L1

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_space_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _case(lens, s_q, n_new, causal=True, cache_dtype="bf16", seed=80):
    wl = mw.make(len(lens), s_q, 128, lens, causal=causal, cache_dtype=cache_dtype, seed=seed, name="var6")
    g = torch.Generator().manual_seed(seed + 1)
    b, h = wl.batch, wl.num_heads
    q = torch.randn(b, s_q, h, 192, generator=g).to(torch.bfloat16)
    k_new = torch.randn(b, n_new, h, 128, generator=g).to(torch.bfloat16)
    v_new = torch.randn(b, n_new, h, 128, generator=g).to(torch.bfloat16)
    wv = mw.make_projections(1, h, seed=seed + 2).w_kvb2
    return wl, q, k_new, v_new, wv


def _run(wl, q, k_new, v_new, wv, n_new):
    shape = mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages, wl.cache_dtype, wl.causal)
    dec = mla.Var6Decoder(shape, n_new)
    out = torch.full((wl.batch, wl.s_q, wl.num_heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.batch, wl.s_q, wl.num_heads), float("nan"), dtype=torch.float32, device="cuda")
    dec.decode(wl.q.cuda(), q.cuda(), wl.pool.cuda(), torch.from_numpy(wl.block_table).cuda(),
               torch.from_numpy(wl.seqlens).cuda(), k_new.cuda(), v_new.cuda(), wv.cuda(), wl.softmax_scale, out, lse,
               kv_scale=None if wl.kv_scale is None else wl.kv_scale.cuda())
    torch.cuda.synchronize()
    assert dec.status() == 0
    return oracle.bf16_to_f64(out.cpu()), lse.cpu().numpy().astype(np.float64)


def _reference(wl, q, k_new, v_new, wv, n_new, rows=None):
    f = oracle.bf16_to_f64
    return oracle.mlavar6_decode(wl, f(wl.q), f(q), f(k_new), f(v_new), f(wv), n_new, rows=rows)


def _assert_contract(got, L, ref, Lr):
    assert np.all(np.isfinite(got))
    assert np.array_equal(np.isneginf(L), np.isneginf(Lr))
    fin = np.isfinite(Lr)
    if fin.any():
        assert np.max(np.abs(L[fin] - Lr[fin])) <= LSE_MAX_ABS
    rr = oracle.round_bf16(ref)
    assert np.max(np.abs(got - ref)) <= O_MAX_ABS
    den = np.abs(rr).sum()
    rel = np.abs(got - rr).sum() / den if den > 0 else np.abs(got).sum()
    assert rel <= O_REL_L1, rel


def _check(wl, q, k_new, v_new, wv, n_new):
    got, L = _run(wl, q, k_new, v_new, wv, n_new)
    ref, Lr = _reference(wl, q, k_new, v_new, wv, n_new)
    _assert_contract(got, L, ref, Lr)


@pytest.mark.parametrize("n_new", [4, 64, 100])
def test_var6_causal_speculative(n_new):
    _check(*_case([300, 1000], 4, n_new), n_new)


def test_var6_latent_only_and_short_requests():
    # n = 0 is the latent path decompressed; n = 64 > t = 50 leaves the first
    # request with new tokens only
    _check(*_case([300, 700], 4, 0, causal=False, seed=81), 0)
    _check(*_case([50, 700], 4, 64, seed=82), 64)


def test_var6_fp8_cache_and_non_causal():
    _check(*_case([300, 130], 2, 16, cache_dtype="fp8", seed=83), 16)
    _check(*_case([500, 64, 1], 1, 32, causal=False, seed=84), 32)


def test_var6_spec_shape_sampled():
    """The speculative workload's shape (b=32, s=16, t=4096, n=64), checked
    on sampled query tokens of three requests, every head (the oracle
    decompresses every old token's value per head: about 0.5 GFLOP a
    (token, head), so the whole batch is out of its reach)."""
    n = 64
    wl, q, k_new, v_new, wv = _case([4096] * 32, 16, n, seed=85)
    got, L = _run(wl, q, k_new, v_new, wv, n)
    rows = [(0, 0), (0, 15), (13, 7), (31, 15)]
    ref, Lr = _reference(wl, q, k_new, v_new, wv, n, rows=rows)
    _assert_contract(np.stack([got[r, i] for r, i in rows]), np.stack([L[r, i] for r, i in rows]), ref, Lr)
