"""Shared helpers for the GPU parity tests: move a workload to the device,
run the library through its C ABI, and compare with the fp64 oracle using
the tolerances of the decode contract:

  * O (bf16): max |err| <= 2e-2, and relative L1 error against the
    bf16-rounded oracle, sum|o - bf16(o_ref)| / sum|bf16(o_ref)|, <= 1e-3;
  * lse (fp32): max |err| <= 1e-3 against the fp64 oracle.
"""
import ctypes
import os

import numpy as np
import torch

import mla_latent_space_b200 as mla
import oracle

O_MAX_ABS = 2e-2
O_REL_L1 = 1e-3
LSE_MAX_ABS = 1e-3


_test_lib = None


def test_lib():
    """The test library (libmla_b200_test.so): the product's objects plus the
    entry points declared in csrc/test_entry.h."""
    global _test_lib
    if _test_lib is None:
        path = os.path.join(os.path.dirname(mla.LIB_PATH), "libmla_b200_test.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m mla_latent_space_b200.build`")
        L = ctypes.CDLL(path)
        vp, sz, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
        dec = [ctypes.POINTER(mla.mla_shape_t), vp, vp, vp, vp, vp, f32, vp, vp, sz, vp, vp, vp]
        for name in ("mla_decode_fwd_simt", "mla_test_decode_stalled"):
            getattr(L, name).argtypes = dec
            getattr(L, name).restype = ctypes.c_int
        _test_lib = L
    return _test_lib


def mla_decode_fwd_simt(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace, out,
                        lse, stream=None):
    """The SIMT decode kernel of the test library, same arguments as
    mla.mla_decode_fwd."""
    mla._decode_common(test_lib().mla_decode_fwd_simt, "mla_decode_fwd_simt", shape, q, kv_cache, kv_scale,
                       block_table, seqlens, softmax_scale, sched, workspace, out, lse, stream)


def mla_test_decode_stalled(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace,
                            out, lse, stream=None):
    """mla_decode_fwd with the kernel's stall hook: one bounded wait runs out."""
    mla._decode_common(test_lib().mla_test_decode_stalled, "mla_test_decode_stalled", shape, q, kv_cache, kv_scale,
                       block_table, seqlens, softmax_scale, sched, workspace, out, lse, stream)


def to_device(wl, device="cuda"):
    d = dict(q=wl.q.to(device), pool=wl.pool.to(device),
             kv_scale=None if wl.kv_scale is None else wl.kv_scale.to(device),
             block_table=torch.from_numpy(wl.block_table).to(device),
             seqlens=torch.from_numpy(wl.seqlens).to(device))
    return d


def shape_of(wl):
    return mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages, wl.cache_dtype, wl.causal)


def run(wl, dev=None, simt=False, n_sms=None, poison_out=True):
    """Schedule + decode + combine on the GPU; returns (O, lse) on the CPU."""
    dev = to_device(wl) if dev is None else dev
    shape = shape_of(wl)
    dec = mla.Decoder(shape, n_sms=n_sms)
    out = torch.empty((wl.batch, wl.s_q, wl.num_heads, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.batch, wl.s_q, wl.num_heads), dtype=torch.float32, device="cuda")
    if poison_out:
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
    dec.schedule(dev["seqlens"])
    dec.decode(dev["q"], dev["pool"], dev["kv_scale"], dev["block_table"], dev["seqlens"], wl.softmax_scale,
               out, lse, decode_fn=mla_decode_fwd_simt if simt else None)
    torch.cuda.synchronize()
    status = dec.status()
    return out.float().cpu().numpy(), lse.cpu().numpy(), status


def compare(O, L, O_ref, L_ref):
    """Error metrics of the contract; returns a dict."""
    Oq = oracle.round_bf16(O_ref)
    err = np.abs(O.astype(np.float64) - O_ref)
    finite = np.isfinite(L_ref)
    lerr = np.abs(L.astype(np.float64)[finite] - L_ref[finite]) if finite.any() else np.zeros(1)
    den = np.abs(Oq).sum()
    return dict(max_abs=float(err.max()) if err.size else 0.0,
                rel_l1=float(np.abs(O.astype(np.float64) - Oq).sum() / den) if den > 0 else float(np.abs(O).sum()),
                rel_l1_unrounded=float(err.sum() / max(np.abs(O_ref).sum(), 1e-300)),
                lse_max_abs=float(lerr.max()),
                lse_inf_match=bool(np.array_equal(np.isneginf(L), np.isneginf(L_ref))),
                finite=bool(np.isfinite(O).all()))


def assert_parity(m, where=""):
    assert m["finite"], f"{where}: non-finite output {m}"
    assert m["max_abs"] <= O_MAX_ABS, f"{where}: {m}"
    assert m["rel_l1"] <= O_REL_L1, f"{where}: {m}"
    assert m["lse_max_abs"] <= LSE_MAX_ABS, f"{where}: {m}"
    assert m["lse_inf_match"], f"{where}: {m}"


def check_full(wl, **kw):
    O, L, st = run(wl, **kw)
    O_ref, L_ref = oracle.decode(wl)
    m = compare(O, L, O_ref, L_ref)
    assert_parity(m, wl.name)
    assert st == 0, f"device status {st}"
    return m
