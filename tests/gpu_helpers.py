"""Shared helpers for the GPU parity tests: move a workload to the device,
run the library through its C ABI, and compare with the fp64 oracle using
the tolerances of the decode contract:

  * O (bf16): max |err| <= 2e-2, and relative L1 error against the
    bf16-rounded oracle, sum|o - bf16(o_ref)| / sum|bf16(o_ref)|, <= 1e-3;
  * lse (fp32): max |err| <= 1e-3 against the fp64 oracle.
"""
import numpy as np
import torch

import mla_latent_space_b200 as mla
import oracle

O_MAX_ABS = 2e-2
O_REL_L1 = 1e-3
LSE_MAX_ABS = 1e-3


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
               out, lse, simt=simt)
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


def sample_rows(wl, n, seed=0):
    rng = np.random.default_rng(seed)
    rs = rng.choice(wl.batch, size=min(n, wl.batch), replace=False)
    out = []
    for r in rs:
        out.append((int(r), int(rng.integers(wl.s_q))))
    # always include the longest and the shortest request
    for r in (int(np.argmax(wl.seqlens)), int(np.argmin(wl.seqlens))):
        out.append((r, wl.s_q - 1))
    return sorted(set(out))


def check_sampled(wl, n=6, **kw):
    O, L, st = run(wl, **kw)
    rows = sample_rows(wl, n)
    O_ref, L_ref = oracle.decode(wl, rows=rows)
    Og = np.stack([O[r, i] for r, i in rows])
    Lg = np.stack([L[r, i] for r, i in rows])
    m = compare(Og, Lg, O_ref, L_ref)
    assert_parity(m, wl.name)
    assert np.isfinite(O).all(), "non-finite values outside the sampled rows"
    assert st == 0, f"device status {st}"
    return m
