"""GPU parity of the tensor-core projections on either side of the latent
decode (mla_absorb_q, mla_decompress_o, through the C ABI) against the fp64
oracle, and of the whole MLA decode attention they form with the decode:
absorb -> schedule -> decode -> combine -> decompress.

Tolerance of one projection, derived from its arithmetic: the kernel
accumulates K products of bf16 values in fp32 and rounds the sum to bf16, so
against the exact sum x it is off by at most the bf16 rounding (bf16 keeps 8
significant bits, so half an ulp is at most 2^-8 |x|) plus the fp32
accumulation error (bounded by K * 2^-24 * sum |a_k b_k|; the test allows 4x
that for the tensor core's summation order).  Against the bf16-rounded
oracle only rare one-ulp rounding flips may differ: relative L1 <= 1e-4.  The RoPE part of the absorbed
query is a copy and must be bit-exact.
"""
import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
import mla_workloads as mw
import oracle
from gpu_helpers import O_MAX_ABS, O_REL_L1, LSE_MAX_ABS

pytestmark = pytest.mark.gpu

NAN_BF16 = -1   # 0xFFFF: a bf16 NaN, as int16


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_space_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _f64(t):
    return oracle.bf16_to_f64(t.cpu())


def _check_projection(got, ref, absref, K):
    got = _f64(got)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 4 * K * 2.0 ** -24 * absref
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} elements beyond the bound; worst excess {float((err - bound).max())}"
    rr = oracle.round_bf16(ref)
    rel_l1 = np.abs(got - rr).sum() / np.abs(rr).sum()
    assert rel_l1 <= 1e-4, rel_l1          # only rare one-ulp rounding flips may differ
    return float(rel_l1)


def _poisoned(shape, extra_rows):
    """bf16 buffer with `extra_rows` guard rows after the real ones, all NaN."""
    buf = torch.empty((shape[0] + extra_rows,) + tuple(shape[1:]), dtype=torch.bfloat16, device="cuda")
    buf.view(torch.int16).fill_(NAN_BF16)
    return buf


# rows x heads: one row, one head; the decode batch of the DeepSeek-V3
# workload at full size (64 x 128); ragged row tiles (130, 300, 513) over a
# few heads
SHAPES = [(1, 1), (64, 128), (130, 3), (300, 2), (513, 4)]


@pytest.mark.parametrize("rows,heads", SHAPES)
def test_absorb_matches_oracle(rows, heads):
    p = mw.make_projections(rows, heads, seed=rows + heads)
    q, wk = p.q.cuda(), p.w_k.cuda()
    buf = _poisoned((rows, heads, 576), 2)
    qz = buf[:rows]
    mla.mla_absorb_q(q, wk, qz)
    torch.cuda.synchronize()
    qf, wf = _f64(p.q), _f64(p.w_k)
    ref = oracle.absorb(qf, wf)
    absref = oracle.absorb(np.abs(qf), np.abs(wf))
    _check_projection(qz[..., :512], ref[..., :512], absref[..., :512], 128)
    assert torch.equal(qz[..., 512:].cpu().view(torch.int16), p.q[..., 128:].view(torch.int16))
    assert bool((buf[rows:].view(torch.int16) == NAN_BF16).all()), "rows past the end were written"


@pytest.mark.parametrize("rows,heads", SHAPES)
def test_decompress_matches_oracle(rows, heads):
    p = mw.make_projections(rows, heads, seed=7 * rows + heads)
    o, wv = p.o_lat.cuda(), p.w_kvb2.cuda()
    buf = _poisoned((rows, heads, 128), 2)
    out = buf[:rows]
    mla.mla_decompress_o(o, wv, out)
    torch.cuda.synchronize()
    of, wf = _f64(p.o_lat), _f64(p.w_kvb2)
    _check_projection(out, oracle.decompress(of, wf), oracle.decompress(np.abs(of), np.abs(wf)), 512)
    assert bool((buf[rows:].view(torch.int16) == NAN_BF16).all()), "rows past the end were written"


def test_projections_zero_rows():
    p = mw.make_projections(0, 4)
    qz = torch.empty((0, 4, 576), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    mla.mla_absorb_q(p.q.cuda(), p.w_k.cuda(), qz)
    mla.mla_decompress_o(p.o_lat.cuda(), p.w_kvb2.cuda(), out)
    torch.cuda.synchronize()


def test_projections_leave_status_clear():
    p = mw.make_projections(64, 8, seed=2)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_absorb_q(p.q.cuda(), p.w_k.cuda(), torch.empty((64, 8, 576), dtype=torch.bfloat16, device="cuda"),
                     device_status=st)
    mla.mla_decompress_o(p.o_lat.cuda(), p.w_kvb2.cuda(),
                         torch.empty((64, 8, 128), dtype=torch.bfloat16, device="cuda"), device_status=st)
    assert int(st.item()) == 0


@pytest.mark.parametrize("lens", [[300, 64], [1, 4096, 129]])
def test_whole_mla_decode_attention(lens):
    """absorb -> decode -> decompress on the GPU against the same chain in the
    oracle, which rounds its own intermediates to bf16 where the library's
    interface holds bf16 tensors (the absorbed query and the latent output),
    so that the comparison carries the decode's parity bar."""
    b, h = len(lens), 128
    wl = mw.make(b, 1, h, lens, seed=21, name=f"chain{lens}")
    p = mw.make_projections(b, h, seed=22)
    # oracle chain
    qz_ref = oracle.round_bf16(oracle.absorb(_f64(p.q), _f64(p.w_k)))            # [b, h, 576]
    wl.q = torch.from_numpy(qz_ref.reshape(b, 1, h, 576)).to(torch.bfloat16)      # exact: values are bf16
    O_ref, L_ref = oracle.decode(wl)
    out_ref = oracle.decompress(oracle.round_bf16(O_ref[:, 0]), _f64(p.w_kvb2))   # [b, h, 128]
    # GPU chain, every step through the C ABI
    dev = dict(pool=wl.pool.cuda(), block_table=torch.from_numpy(wl.block_table).cuda(),
               seqlens=torch.from_numpy(wl.seqlens).cuda())
    qz = torch.empty((b, 1, h, 576), dtype=torch.bfloat16, device="cuda")
    mla.mla_absorb_q(p.q.cuda().view(b, 1, h, 192), p.w_k.cuda(), qz)
    shape = mla.make_shape(b, 1, h, wl.max_pages, wl.num_pages)
    dec = mla.Decoder(shape)
    o_lat = torch.empty((b, 1, h, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((b, 1, h), dtype=torch.float32, device="cuda")
    dec.schedule(dev["seqlens"])
    dec.decode(qz, dev["pool"], None, dev["block_table"], dev["seqlens"], wl.softmax_scale, o_lat, lse)
    out = torch.empty((b, 1, h, 128), dtype=torch.bfloat16, device="cuda")
    mla.mla_decompress_o(o_lat, p.w_kvb2.cuda(), out)
    torch.cuda.synchronize()
    assert dec.status() == 0
    assert np.max(np.abs(lse.cpu().numpy().astype(np.float64) - L_ref)) <= LSE_MAX_ABS
    got = _f64(out)[:, 0]
    assert np.all(np.isfinite(got))
    rr = oracle.round_bf16(out_ref)
    assert np.max(np.abs(got - out_ref)) <= O_MAX_ABS
    rel_l1 = np.abs(got - rr).sum() / np.abs(rr).sum()
    assert rel_l1 <= O_REL_L1, rel_l1
