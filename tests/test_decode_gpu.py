"""GPU parity of the decode path (schedule -> decode -> combine through the
C ABI) against the fp64 oracle, on the five workloads and their edge cases.
"""
import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
import mla_workloads as mw
import oracle
from gpu_helpers import (assert_parity, check_full, compare, mla_test_decode_stalled, run, shape_of,
                         to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_space_b200 import build
    build.build()
    assert torch.cuda.is_available()


# ---- small cases the oracle finishes in seconds ---------------------------

def test_config1_tiny_full():
    check_full(mw.make_config(1))


@pytest.mark.parametrize("lens", [[1], [63, 64, 65], [700, 1, 129, 4096], [0, 77]])
def test_ragged_lengths_h128(lens):
    check_full(mw.make(len(lens), 1, 128, lens, seed=11, name=f"ragged{lens}"))


def test_small_jagged_h128():
    check_full(mw.make(6, 1, 128, None, jagged=(128, 3000), seed=4, name="jagged_small"))


def test_small_fp8():
    check_full(mw.make(3, 1, 128, [300, 64, 1000], cache_dtype="fp8", seed=5, name="fp8_small"))


def test_small_causal_spec():
    check_full(mw.make(3, 16, 128, [200, 16, 700], causal=True, seed=6, name="spec_small"))


@pytest.mark.parametrize("h,s_q,causal", [(16, 1, False), (64, 2, True), (48, 4, True), (128, 2, False)])
def test_head_counts_and_packed_tiles(h, s_q, causal):
    check_full(mw.make(3, s_q, h, [130, 5, 260], causal=causal, seed=7, name=f"h{h}s{s_q}"))


def test_simt_debug_path_matches_oracle():
    check_full(mw.make(3, 1, 128, [300, 64, 1000], seed=8), simt=True)
    check_full(mw.make(2, 16, 128, [100, 300], causal=True, seed=8), simt=True)


@pytest.mark.parametrize("h,s_q", [(1, 1), (3, 5), (128, 32), (256, 1)])
def test_degenerate_and_large_tile_shapes(h, s_q):
    """One head (a tile of one row), head counts that do not divide a tile,
    32 query tokens (a causal step of 4096 rows per request), and 256 heads
    (two tiles per query token)."""
    check_full(mw.make(2, s_q, h, [max(s_q, 70), max(s_q, 300)], causal=s_q > 1, seed=26, name=f"shape_h{h}s{s_q}"))


def test_many_short_requests():
    """Far more tiles than SM pairs (600 requests of 1..200 tokens): the
    scheduler packs many whole tiles per worker."""
    rng = np.random.default_rng(27)
    check_full(mw.make(600, 1, 128, rng.integers(1, 201, size=600).tolist(), seed=27, name="many_short"))


def test_every_request_empty():
    """No visible key anywhere: every O row is 0 and every lse is -inf."""
    wl = mw.make(3, 2, 128, [0, 0, 0], seed=28, name="all_empty")
    O, L, st = run(wl)
    assert st == 0
    assert np.all(O == 0) and np.all(np.isneginf(L))


@pytest.mark.parametrize("n_sms", [2, 16, 148, 1000])
def test_split_counts_agree(n_sms):
    # the same rows, cut into 1 .. hundreds of pieces, stay within tolerance
    wl = mw.make(4, 1, 128, [3000, 64, 1, 2500], seed=9, name="splits")
    check_full(wl, n_sms=n_sms)


def _growing_scores(name):
    # A RoPE column equal to the token index (query column 1 there) makes the
    # scores grow by softmax_scale * log2(e) ~ 0.10 log2 units per token: each
    # 128-token block's max then exceeds the running max by ~13 > 8, so O is
    # rescaled before nearly every block's PVs.
    wl = mw.make(2, 1, 128, [4096, 1000], seed=12, name=name)
    for r, t in enumerate(wl.seqlens):
        for j in range((int(t) + 63) // 64):
            page = int(wl.block_table[r, j])
            wl.pool[page, :, 512] = torch.arange(64 * j, 64 * j + 64, dtype=torch.float32).to(torch.bfloat16)
    wl.q[..., 512] = 1.0
    return wl


@pytest.mark.parametrize("n_sms", [None, 16])
def test_running_max_rescales_every_block(n_sms):
    # with 16 SMs also across split pieces, whose partials the combine merges
    check_full(_growing_scores("rescale"), n_sms=n_sms)


def test_fp8_running_max_rescales_every_block():
    import dataclasses
    wl = _growing_scores("rescale_fp8")
    pool, ks = mw.quantize_fp8_pages(wl.pool)   # the RoPE part stays bf16
    check_full(dataclasses.replace(wl, pool=pool, kv_scale=ks, cache_dtype="fp8"))


def test_nan_in_unused_slots_and_pages():
    wl = mw.make(3, 1, 128, [70, 130, 1], seed=10, name="poison")
    O0, L0, _ = run(wl)
    for r, t in enumerate(wl.seqlens):
        n = (int(t) + 63) // 64
        last = int(wl.block_table[r, n - 1])
        if t % 64:
            wl.pool[last, int(t) % 64:] = float("nan")
        wl.block_table[r, n:] = 0
    extra = torch.full((2, 64, 576), float("nan"), dtype=torch.bfloat16)
    wl.pool = torch.cat([wl.pool, extra])
    O1, L1, st = run(wl)
    assert st == 0 and np.isfinite(O1).all() and np.array_equal(O0, O1) and np.array_equal(L0, L1)


def test_device_schedule_equals_host_planner():
    import mla_workloads as mw2
    for cfg in (2, 3, 5):
        b, s, h, lens = mw2.config_shape(cfg)
        shape = mla.make_shape(b, s, h, int((lens.max() + 63) // 64), 1, causal=(cfg == 5))
        host = mla.mla_plan_schedule_host(shape, torch.from_numpy(lens), 148)
        dev = torch.empty(host.numel(), dtype=torch.int32, device="cuda")
        mla.mla_get_schedule(shape, torch.from_numpy(lens).cuda(), 148, dev)
        torch.cuda.synchronize()
        assert torch.equal(dev.cpu(), host)


def test_bad_page_id_is_flagged_not_faulted():
    wl = mw.make(2, 1, 128, [100, 100], seed=12)
    wl.block_table[1, 1] = 10 ** 6          # beyond the pool: skipped and flagged
    O, L, st = run(wl)
    assert st == -6                         # MLA_ERR_DEVICE_CHECK
    O_ref, L_ref = oracle.decode(mw.make(2, 1, 128, [100, 100], seed=12))
    assert_parity(compare(O[:1], L[:1], O_ref[:1], L_ref[:1]), "unaffected request")


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """Failure detection without a fault: the test library's stalled decode
    makes one of the kernel's bounded waits wait on a barrier that nothing
    arrives on.  After its 2 s limit the kernel reports MLA_ERR_TIMEOUT
    through the status word, both CTAs of every pair stop, drain and free
    their tensor memory, and the next decode on the same context is at
    parity."""
    import time
    wl = mw.make(2, 1, 128, [300, 100], seed=19, name="stall")
    dev = to_device(wl)
    shape = shape_of(wl)
    dec = mla.Decoder(shape)
    out = torch.empty((2, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 1, 128), dtype=torch.float32, device="cuda")
    dec.schedule(dev["seqlens"])
    t0 = time.perf_counter()
    mla_test_decode_stalled(shape, dev["q"], dev["pool"], None, dev["block_table"], dev["seqlens"], wl.softmax_scale,
                            dec.sched, dec.workspace, out, lse)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert dec.status() == -5                       # MLA_ERR_TIMEOUT
    assert 1.0 < dt < 30.0, dt                      # the wait's own limit ended it
    assert dec.status() == 0                        # reading the status cleared it
    check_full(wl)                                  # the context is still usable


def test_value_beyond_fp16_range_is_flagged():
    """PV runs in fp16: a bf16 value entry of 1e5 cannot be represented.
    The decode flags it (MLA_ERR_DEVICE_CHECK) instead of returning a wrong
    result silently; the request that does not read that page is still at
    parity."""
    wl = mw.make(2, 1, 128, [100, 100], seed=17, name="v_overflow")
    page = int(wl.block_table[1, 0])
    wl.pool[page, 5, 17] = 1e5                  # a value column (< 512) of request 1
    O, L, st = run(wl)
    assert st == -6                             # MLA_ERR_DEVICE_CHECK
    O_ref, L_ref = oracle.decode(wl, rows=[(0, 0)])
    assert_parity(compare(O[:1, 0], L[:1, 0], O_ref, L_ref), "unaffected request")


def test_fp8_value_times_scale_beyond_fp16_range_is_flagged():
    """The FP8 cache's values times their per-token scale enter PV as fp16:
    a scale of 1e3 puts the token's larger e4m3 values above 65504."""
    import dataclasses
    wl = mw.make(2, 1, 128, [100, 100], cache_dtype="fp8", seed=18, name="fp8_v_overflow")
    page = int(wl.block_table[1, 0])
    ks = wl.kv_scale.clone()
    ks[page, 9] = 1e3
    wl = dataclasses.replace(wl, kv_scale=ks)
    O, L, st = run(wl)
    assert st == -6
    O_ref, L_ref = oracle.decode(wl, rows=[(0, 0)])
    assert_parity(compare(O[:1, 0], L[:1, 0], O_ref, L_ref), "unaffected request")


# ---- the five workloads at full size, every row ------------------------------

@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_configs_every_row(cfg):
    """Configs 2-5 at their full sizes, the launch configuration the bench
    times: every O element and every LSE of the batch against the oracle
    (which gathers one request's cache at a time, so the 131072-token
    requests of the jagged batch stay within a few hundred MB)."""
    check_full(mw.make_config(cfg))


# ---- FP8 cache: the kFp8 kernel across the same edge cases ------------------

def test_fp8_query_beyond_fp16_range():
    """The FP8 kernel's latent scores use a two-part e4m3 copy of the query
    with a per-row power-of-two scale, so query values far outside fp16's
    range are as good as any: q * 2^17 with softmax_scale / 2^17 is the same
    problem (both scalings are exact)."""
    wl = mw.make(2, 1, 128, [300, 70], cache_dtype="fp8", seed=71, name="fp8_big_query")
    wl.q = (wl.q.float() * 2.0 ** 17).to(torch.bfloat16)
    assert float(wl.q.float().abs().max()) > 65504.0
    wl.softmax_scale = wl.softmax_scale / 2.0 ** 17
    check_full(wl)


def test_fp8_query_far_below_normal_range():
    """The other end: q * 2^-122 with softmax_scale * 2^122.  The row's
    power-of-two scale would be 2^-128; it is held at 2^-126 so that its
    inverse stays finite, and the e4m3 split still covers the row."""
    wl = mw.make(2, 1, 128, [300, 70], cache_dtype="fp8", seed=73, name="fp8_tiny_query")
    wl.q = (wl.q.float() * 2.0 ** -122).to(torch.bfloat16)
    wl.softmax_scale = wl.softmax_scale * 2.0 ** 122
    check_full(wl)


def test_fp8_query_rows_of_different_magnitudes():
    # each head's row scaled by its own power of two, 2^-5 .. 2^2 (larger
    # logits would test fp32 accumulation, not the split): every row gets
    # its own scale for the e4m3 split
    wl = mw.make(2, 1, 128, [500, 129], cache_dtype="fp8", seed=72, name="fp8_row_scales")
    f = torch.tensor([2.0 ** (j % 8 - 5) for j in range(128)])
    wl.q = (wl.q.float() * f[None, None, :, None]).to(torch.bfloat16)
    check_full(wl)


def test_fp8_causal_spec_and_packed_tiles():
    check_full(mw.make(3, 16, 128, [200, 16, 700], causal=True, cache_dtype="fp8", seed=13, name="fp8_spec"))
    check_full(mw.make(3, 2, 64, [130, 5, 260], causal=True, cache_dtype="fp8", seed=14, name="fp8_h64s2"))


@pytest.mark.parametrize("n_sms", [2, 16, 1000])
def test_fp8_split_counts_agree(n_sms):
    wl = mw.make(4, 1, 128, [3000, 64, 1, 2500], cache_dtype="fp8", seed=15, name="fp8_splits")
    check_full(wl, n_sms=n_sms)


def test_fp8_nan_in_unused_slots_and_pages():
    """e4m3 NaN bytes, bf16 NaN RoPE values and NaN scales past each
    request's length, and unused block-table slots pointing at NaN pages,
    change nothing."""
    wl = mw.make(3, 1, 128, [70, 130, 1], cache_dtype="fp8", seed=16, name="fp8_poison")
    O0, L0, _ = run(wl)
    pool = wl.pool.clone()
    scale = wl.kv_scale.clone()
    nan_bf16 = torch.tensor([float("nan")], dtype=torch.bfloat16).view(torch.uint8)   # 2 bytes
    for r, t in enumerate(wl.seqlens):
        n = (int(t) + 63) // 64
        last = int(wl.block_table[r, n - 1])
        for tok in range(int(t) % 64 if t % 64 else 64, 64):
            pool[last, tok * 512:(tok + 1) * 512] = 0x7F                       # e4m3 NaN
            rope = pool[last, 64 * 512 + tok * 128:64 * 512 + (tok + 1) * 128].view(-1, 2)
            rope[:] = nan_bf16
            scale[last, tok] = float("nan")
        wl.block_table[r, n:] = wl.num_pages                                   # the extra NaN page
    extra = torch.full((1, pool.shape[1]), 0x7F, dtype=torch.uint8)
    wl.pool = torch.cat([pool, extra])
    wl.kv_scale = torch.cat([scale, torch.full((1, 64), float("nan"))])
    O1, L1, st = run(wl)
    assert st == 0 and np.isfinite(O1).all() and np.array_equal(O0, O1) and np.array_equal(L0, L1)
