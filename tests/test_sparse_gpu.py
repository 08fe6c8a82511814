"""GPU parity of the token-level sparse decode (mla_sparse_decode_fwd through
the C ABI) against the fp64 oracle, with the decode's tolerances: O max|err|
<= 2e-2 and relative L1 against the bf16-rounded oracle <= 1e-3; lse max|err|
<= 1e-3.
"""
import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
import mla_workloads as mw
import oracle
from gpu_helpers import assert_parity, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_space_b200 import build
    build.build()
    assert torch.cuda.is_available()


def run_sparse(wl, idx, poison_out=True):
    shape = mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages, wl.cache_dtype)
    dec = mla.SparseDecoder(shape, idx.shape[-1])
    out = torch.empty((wl.batch, wl.s_q, wl.num_heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.batch, wl.s_q, wl.num_heads), dtype=torch.float32, device="cuda")
    if poison_out:
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
    dec.decode(wl.q.cuda(), wl.pool.cuda(), torch.from_numpy(wl.block_table).cuda(),
               torch.from_numpy(wl.seqlens).cuda(), torch.from_numpy(idx).cuda(), wl.softmax_scale, out, lse,
               kv_scale=None if wl.kv_scale is None else wl.kv_scale.cuda())
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), dec.status()


def check(wl, idx):
    O, L, st = run_sparse(wl, idx)
    assert st == 0, mla.error_string(st)
    O_ref, L_ref = oracle.sparse_decode(wl, idx)
    m = compare(O, L, O_ref, L_ref)
    assert_parity(m, wl.name)
    return m


def test_sparse_random_lists_with_padding_duplicates_and_out_of_range():
    wl = mw.make(3, 2, 128, [300, 70, 1000], seed=31, name="sparse_small")
    idx = mw.make_sparse_indices(wl.seqlens, 2, 100, seed=32, pad=10)
    idx[0, 0, 95] = idx[0, 0, 3]           # a repeated position
    idx[1, 1, 96] = 70                      # one past the end: skipped
    idx[2, 0, 97] = -5                      # negative: skipped
    idx[2, 1, 98] = 999                     # the last token
    check(wl, idx)


@pytest.mark.parametrize("topk", [1, 63, 64, 65, 300])
def test_sparse_list_lengths(topk):
    # ragged virtual pages: the compacted lengths span one page, its edge, and several pages
    wl = mw.make(2, 1, 128, [500, 4000], seed=33, name=f"sparse_k{topk}")
    check(wl, mw.make_sparse_indices(wl.seqlens, 1, topk, seed=34))


def test_sparse_every_position_equals_the_dense_decode_oracle():
    wl = mw.make(2, 1, 128, [130, 64], seed=35, name="sparse_dense")
    idx = np.full((2, 1, 140), -1, dtype=np.int32)
    for r, t in enumerate(wl.seqlens):
        idx[r, 0, :t] = np.arange(t)
    O, L, st = run_sparse(wl, idx)
    assert st == 0
    O_ref, L_ref = oracle.decode(wl)
    assert_parity(compare(O, L, O_ref, L_ref), "sparse_dense")


def test_sparse_empty_lists_and_nan_outside_the_lists():
    # rows that no list names are NaN, so any read of them would show
    wl = mw.make(2, 1, 128, [200, 90], seed=36, name="sparse_poison")
    idx = mw.make_sparse_indices(wl.seqlens, 1, 40, seed=37)
    idx[1] = -1                              # request 1: nothing valid -> O = 0, lse = -inf
    named = {(r, int(j)) for r in range(2) for j in idx[r, 0] if j >= 0}
    for r, t in enumerate(wl.seqlens):
        for j in range(int(t)):
            if (r, j) not in named:
                wl.pool[int(wl.block_table[r][j // 64]), j % 64] = float("nan")
    O, L, st = run_sparse(wl, idx)
    assert st == 0
    O_ref, L_ref = oracle.sparse_decode(wl, idx)
    assert_parity(compare(O, L, O_ref, L_ref), "sparse_poison")
    assert np.all(O[1] == 0) and np.all(np.isneginf(L[1]))


def test_sparse_bench_shape_sampled():
    """The bench's shape (b=64, t=32768, 2048 positions per query token), in
    the launch configuration the bench times, checked on 6 sampled requests."""
    wl = mw.make(64, 1, 128, 32768, seed=40, name="sparse_b64_t32768_k2048")
    idx = mw.make_sparse_indices(wl.seqlens, 1, 2048, seed=41)
    O, L, st = run_sparse(wl, idx)
    assert st == 0
    rs = [0, 17, 31, 42, 55, 63]
    sub = mw.Workload(name="sub", batch=len(rs), s_q=1, num_heads=128, causal=False, cache_dtype="bf16",
                      seqlens=wl.seqlens[rs], block_table=wl.block_table[rs], q=wl.q[rs], pool=wl.pool,
                      kv_scale=None, softmax_scale=wl.softmax_scale)
    O_ref, L_ref = oracle.sparse_decode(sub, idx[rs])
    assert_parity(compare(O[rs], L[rs], O_ref, L_ref), "sparse_bench_sampled")


def test_sparse_fp8_random_lists_with_padding_and_out_of_range():
    wl = mw.make(3, 2, 128, [300, 70, 1000], cache_dtype="fp8", seed=61, name="sparse_fp8")
    idx = mw.make_sparse_indices(wl.seqlens, 2, 100, seed=62, pad=10)
    idx[0, 1, 90] = idx[0, 1, 0]            # a repeated position
    idx[1, 0, 91] = 70                      # one past the end: skipped
    idx[2, 1, 92] = 999                     # the last token
    check(wl, idx)


@pytest.mark.parametrize("topk", [1, 65, 700])
def test_sparse_fp8_list_lengths(topk):
    wl = mw.make(2, 1, 128, [500, 4000], cache_dtype="fp8", seed=63, name=f"sparse_fp8_k{topk}")
    check(wl, mw.make_sparse_indices(wl.seqlens, 1, topk, seed=64))
