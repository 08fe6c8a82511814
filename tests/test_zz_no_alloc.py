"""The no-allocation entry point, mla_decode_fwd_noalloc: the whole decode
step with the library's static scratch.  Collected last on purpose (the
static scratch outlives every other test in the process), and written to
pass alone as well.

Each case runs the existing path (mla_get_schedule -> mla_decode_fwd ->
mla_combine with torch-allocated buffers) and the no-allocation path on the
same inputs, twice in a row with different workloads, and checks both
against the fp64 oracle with the decode contract's tolerances; the two
paths split the work differently, so they agree to rounding, not bit for
bit.
"""
import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
import mla_workloads as mw
import oracle
from gpu_helpers import assert_parity, compare, run, shape_of, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_space_b200 import build
    build.build()
    assert torch.cuda.is_available()


def run_noalloc(wl, dev=None):
    dev = to_device(wl) if dev is None else dev
    shape = shape_of(wl)
    out = torch.full((wl.batch, wl.s_q, wl.num_heads, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.batch, wl.s_q, wl.num_heads), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    mla.mla_decode_fwd_noalloc(shape, dev["q"], dev["pool"], dev["kv_scale"], dev["block_table"], dev["seqlens"],
                               wl.softmax_scale, out, lse, device_status=status)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(status.item())


WORKLOADS = [
    # ragged lengths incl. an empty request and page-boundary cases, h=128
    lambda: mw.make(5, 1, 128, [0, 1, 64, 65, 700], seed=21, name="noalloc_ragged"),
    # several tiles per request (s_q=2, h=128), causal, jagged lengths
    lambda: mw.make(4, 2, 128, None, jagged=(64, 2000), causal=True, seed=22, name="noalloc_spec"),
    # small heads, contiguous pages (config 1 shape)
    lambda: mw.make_config(1),
    # fp8 cache
    lambda: mw.make(3, 1, 128, [300, 64, 1000], cache_dtype="fp8", seed=23, name="noalloc_fp8"),
]


@pytest.mark.parametrize("first,second", [(0, 1), (2, 3), (1, 0)])
def test_two_calls_in_a_row_match_existing_entry_point(first, second):
    for k in (first, second):
        wl = WORKLOADS[k]()
        dev = to_device(wl)
        O_ref, L_ref = oracle.decode(wl)
        O_a, L_a, st_a = run(wl, dev=dev)                 # existing entry point
        O_b, L_b, st_b = run_noalloc(wl, dev=dev)         # no-allocation entry point
        assert st_a == 0 and st_b == 0, (st_a, st_b)
        assert_parity(compare(O_a, L_a, O_ref, L_ref), wl.name + " (existing)")
        assert_parity(compare(O_b, L_b, O_ref, L_ref), wl.name + " (noalloc)")
        # the two paths agree to rounding
        assert np.abs(O_a - O_b).max() <= 2e-2, wl.name
        fin = np.isfinite(L_a)
        assert np.array_equal(fin, np.isfinite(L_b)), wl.name
        assert np.abs(L_a[fin] - L_b[fin]).max(initial=0.0) <= 1e-3, wl.name


def test_device_status_reports_bad_page_ids():
    wl = mw.make(2, 1, 128, [200, 100], seed=24, name="noalloc_badpage")
    dev = to_device(wl)
    dev["block_table"][1, 0] = wl.num_pages + 5          # out of range: skipped and flagged
    _, _, st = run_noalloc(wl, dev=dev)
    assert st != 0
    # the next call starts from a cleared status word
    wl2 = mw.make(2, 1, 128, [200, 100], seed=25, name="noalloc_after_bad")
    _, _, st2 = run_noalloc(wl2)
    assert st2 == 0
