"""The decode step (schedule -> decode -> combine) and the whole MLA decode
attention (absorb -> schedule -> decode -> combine -> decompress) captured
once in a CUDA graph and replayed on new query values, against the fp64
oracle.  Every launch goes through the C ABI during capture; the replays
reuse the captured tensor maps and buffers, so only the tensor contents may
change between replays.
"""
import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
import mla_workloads as mw
import oracle
from gpu_helpers import O_MAX_ABS, O_REL_L1, LSE_MAX_ABS, assert_parity, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_space_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _new_q(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def test_decode_step_replays_from_a_cuda_graph():
    wl = mw.make(4, 1, 128, [300, 1000, 64, 2000], seed=50, name="graph")
    shape = mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages)
    dec = mla.Decoder(shape)
    q = wl.q.cuda()
    pool, bt = wl.pool.cuda(), torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seqlens).cuda()
    out = torch.empty((wl.batch, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.batch, 1, 128), dtype=torch.float32, device="cuda")

    def step():
        dec.schedule(sl)
        dec.decode(q, pool, None, bt, sl, wl.softmax_scale, out, lse)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                      # first calls (attributes, device queries) outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in (51, 52):
        wl.q = _new_q(tuple(wl.q.shape), seed)
        q.copy_(wl.q)
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert dec.status() == 0
        O_ref, L_ref = oracle.decode(wl)
        assert_parity(compare(out.float().cpu().numpy(), lse.cpu().numpy(), O_ref, L_ref), f"graph replay {seed}")


def test_whole_attention_replays_from_a_cuda_graph():
    b, h = 3, 128
    wl = mw.make(b, 1, h, [500, 129, 2048], seed=53, name="graph_chain")
    p = mw.make_projections(b, h, seed=54)
    shape = mla.make_shape(b, 1, h, wl.max_pages, wl.num_pages)
    dec = mla.Decoder(shape)
    qin = p.q.cuda().view(b, 1, h, 192)
    wk, wv = p.w_k.cuda(), p.w_kvb2.cuda()
    pool, bt = wl.pool.cuda(), torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seqlens).cuda()
    qz = torch.empty((b, 1, h, 576), dtype=torch.bfloat16, device="cuda")
    lat = torch.empty((b, 1, h, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((b, 1, h), dtype=torch.float32, device="cuda")
    out = torch.empty((b, 1, h, 128), dtype=torch.bfloat16, device="cuda")

    def chain():
        mla.mla_absorb_q(qin, wk, qz)
        dec.schedule(sl)
        dec.decode(qz, pool, None, bt, sl, wl.softmax_scale, lat, lse)
        mla.mla_decompress_o(lat, wv, out)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        chain()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain()
    qnew = _new_q((b, h, 192), 55)
    qin.copy_(qnew.view(b, 1, h, 192))
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert dec.status() == 0
    f64 = lambda t: oracle.bf16_to_f64(t.cpu())
    qz_ref = oracle.round_bf16(oracle.absorb(f64(qnew), f64(p.w_k)))
    wl.q = torch.from_numpy(qz_ref.reshape(b, 1, h, 576)).to(torch.bfloat16)
    O_ref, L_ref = oracle.decode(wl)
    out_ref = oracle.decompress(oracle.round_bf16(O_ref[:, 0]), f64(p.w_kvb2))
    got = f64(out)[:, 0]
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(lse.cpu().numpy().astype(np.float64) - L_ref)) <= LSE_MAX_ABS
    rr = oracle.round_bf16(out_ref)
    assert np.max(np.abs(got - out_ref)) <= O_MAX_ABS
    assert np.abs(got - rr).sum() / np.abs(rr).sum() <= O_REL_L1
