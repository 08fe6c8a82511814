"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/mla.h declares, sizes its buffers, and rejects bad
arguments before launching anything.  The scheduler's host copy (the same
code as the device kernel) is checked for exact coverage and balance."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import mla_latent_space_b200 as mla
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "mla.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", src)))


def test_library_builds_and_exports_every_declared_symbol():
    from mla_latent_space_b200 import build
    build.build()
    L = mla.lib()
    names = _declared()
    assert "mla_decode_fwd" in names and "mla_get_schedule" in names and "mla_combine" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(mla.EXPORTED) <= set(names)
    assert b"sm_100a" in L.mla_version()


def test_error_strings():
    for code in range(0, -7, -1):
        s = mla.error_string(code)
        assert s.startswith("MLA_")
    assert "unknown" in mla.error_string(42)


def _shape(**kw):
    base = dict(batch=2, s_q=1, num_heads=128, max_pages_per_seq=4, num_pages=8)
    base.update(kw)
    return mla.make_shape(**base)


def test_buffer_sizes():
    s = _shape()
    # header 16 + 74 workers x 8 + 2 tiles x 4 int32 words
    assert mla.mla_schedule_bytes(s, 148) == 4 * (16 + 74 * 8 + 2 * 4)
    assert mla.mla_workspace_bytes(s, 148) == 256 + 148 * (128 * 512 * 4 + 128 * 4)
    s5 = _shape(batch=32, s_q=16, num_heads=128, max_pages_per_seq=64)
    assert mla.mla_schedule_bytes(s5, 148) == 4 * (16 + 74 * 8 + 32 * 16 * 4)
    bad = _shape()
    bad.d_qk = 192
    assert mla.mla_schedule_bytes(bad, 148) == 0


def _call_decode(shape, **over):
    fake = ctypes.c_void_p(1 << 20)     # never dereferenced: validation fails first
    args = dict(q=fake, kv=fake, kv_scale=None, bt=fake, sl=fake, scale=0.07, sched=fake, ws=fake,
                ws_bytes=1 << 20, out=fake, lse=fake)
    args.update(over)
    return mla.lib().mla_decode_fwd(ctypes.byref(shape), args["q"], args["kv"], args["kv_scale"], args["bt"],
                                    args["sl"], args["scale"], args["sched"], args["ws"], args["ws_bytes"],
                                    args["out"], args["lse"], None)


@pytest.mark.parametrize("field,value,code", [
    ("d_qk", 192, -2), ("d_v", 128, -2), ("page_size", 16, -2), ("cache_dtype", 7, -2),
    ("batch", 0, -1), ("s_q", 0, -1), ("num_heads", 0, -1), ("max_pages_per_seq", 0, -1),
    ("num_pages", 0, -1), ("causal", 2, -1)])
def test_decode_rejects_bad_shapes(field, value, code):
    s = _shape()
    setattr(s, field, value)
    assert _call_decode(s) == code


def test_decode_rejects_bad_pointers():
    s = _shape()
    assert _call_decode(s, q=None) == -1
    assert _call_decode(s, out=None) == -1
    assert _call_decode(s, q=ctypes.c_void_p((1 << 20) + 2)) == -1          # q not 16-byte aligned
    assert _call_decode(s, kv=ctypes.c_void_p((1 << 20) + 64)) == -1        # pool not 256-byte aligned
    assert _call_decode(s, ws=ctypes.c_void_p((1 << 20) + 16)) == -1
    assert _call_decode(s, scale=float("nan")) == -1
    assert _call_decode(s, ws_bytes=16) == -3
    s8 = _shape(cache_dtype="fp8")
    assert _call_decode(s8, kv_scale=None) == -1                             # fp8 needs scales


def test_schedule_and_combine_reject_bad_args():
    s = _shape()
    fake = ctypes.c_void_p(1 << 20)
    L = mla.lib()
    assert L.mla_get_schedule(ctypes.byref(s), None, 148, fake, 1 << 20, None) == -1
    assert L.mla_get_schedule(ctypes.byref(s), fake, 148, fake, 16, None) == -3
    assert L.mla_get_schedule(ctypes.byref(s), fake, 0, fake, 1 << 20, None) == -1
    assert L.mla_combine(ctypes.byref(s), None, fake, 1 << 20, fake, fake, None) == -1
    assert L.mla_combine(ctypes.byref(s), fake, fake, 8, fake, fake, None) == -3
    assert L.mla_get_device_status(None, fake, None, None) == -1


def test_sparse_workspace_and_argument_checks():
    s = mla.make_shape(64, 1, 128, 512, 32768)
    # virtual requests: 64 x 32 scratch pages of 73,728 B, plus lengths, block table, schedule, decode workspace
    nb = mla.mla_sparse_workspace_bytes(s, 2048, 148)
    assert 64 * 32 * 73728 < nb < 64 * 32 * 73728 + (64 << 20)
    # FP8: 40,960-byte scratch pages plus 64 fp32 scales per page
    nb8 = mla.mla_sparse_workspace_bytes(mla.make_shape(64, 1, 128, 512, 32768, cache_dtype="fp8"), 2048, 148)
    assert 64 * 32 * (40960 + 256) < nb8 < 64 * 32 * (40960 + 256) + (64 << 20)
    assert mla.mla_sparse_workspace_bytes(mla.make_shape(4, 2, 128, 8, 64, causal=True), 64, 148) == 0
    assert mla.mla_sparse_workspace_bytes(s, 0, 148) == 0
    L = mla.lib()
    fake = ctypes.c_void_p(1 << 20)
    args = lambda sh, k, idx=fake, q=fake, sc=None: (ctypes.byref(sh), k, q, fake, sc, fake, fake, idx, 0.1, fake,
                                                     1 << 40, fake, fake, None)
    assert L.mla_sparse_decode_fwd(*args(s, 2048, idx=None)) == -1
    assert L.mla_sparse_decode_fwd(*args(s, 2048, q=ctypes.c_void_p((1 << 20) + 8))) == -1
    assert L.mla_sparse_decode_fwd(*args(s, 0)) == -1
    assert L.mla_sparse_decode_fwd(*args(mla.make_shape(64, 1, 128, 512, 32768, cache_dtype="fp8"), 2048)) == -1
    assert L.mla_sparse_decode_fwd(*args(mla.make_shape(64, 1, 128, 512, 32768, cache_dtype="fp8"), 2048,
                                         sc=ctypes.c_void_p((1 << 20) + 2))) == -1
    assert L.mla_sparse_decode_fwd(*args(mla.make_shape(4, 2, 128, 8, 64, causal=True), 64)) == -1


def test_var6_workspace_and_argument_checks():
    L = mla.lib()
    s = mla.make_shape(32, 16, 128, 64, 2048, causal=True)
    # old lengths, schedule, decode workspace, then the latent output (two bf16 terms x 512), its lse (fp32)
    # and its decompression (two bf16 terms x 128) for 32 x 16 x 128 rows
    rows = 32 * 16 * 128
    per_row = 2 * 1024 + 4 + 2 * 256
    nb = L.mla_var6_workspace_bytes(ctypes.byref(s), 64, 148)
    assert rows * per_row < nb < rows * per_row + (64 << 20)
    assert L.mla_var6_workspace_bytes(ctypes.byref(s), 8, 148) == 0          # causal needs n >= s_q
    assert L.mla_var6_workspace_bytes(ctypes.byref(mla.make_shape(32, 16, 128, 64, 2048)), 8, 148) > 0
    assert L.mla_var6_workspace_bytes(ctypes.byref(mla.make_shape(2, 33, 128, 64, 2048)), 64, 148) == 0
    assert L.mla_var6_workspace_bytes(ctypes.byref(s), -1, 148) == 0
    fake = ctypes.c_void_p(1 << 20)
    args = lambda sh, n, kn=fake, qz=fake: (ctypes.byref(sh), n, qz, fake, fake, None, fake, fake, kn, fake, fake,
                                            0.1, fake, 1 << 40, fake, fake, None)
    assert L.mla_var6_decode_fwd(*args(s, 8)) == -1                            # causal, n < s_q
    assert L.mla_var6_decode_fwd(*args(s, 64, kn=None)) == -1                  # n > 0 needs k_new
    assert L.mla_var6_decode_fwd(*args(s, 64, qz=ctypes.c_void_p((1 << 20) + 8))) == -1
    assert L.mla_var6_decode_fwd(*args(mla.make_shape(2, 33, 128, 64, 2048), 64)) == -2


def test_projections_reject_bad_args_before_any_launch():
    L = mla.lib()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    for fn in (L.mla_absorb_q, L.mla_decompress_o):
        assert fn(4, 128, None, fake, fake, None, None) == -1
        assert fn(4, 128, fake, None, fake, None, None) == -1
        assert fn(4, 128, fake, fake, None, None, None) == -1
        assert fn(-1, 128, fake, fake, fake, None, None) == -1
        assert fn(4, 0, fake, fake, fake, None, None) == -1
        assert fn(4, 65536, fake, fake, fake, None, None) == -1
        assert fn(4, 128, odd, fake, fake, None, None) == -1                 # 16-byte alignment
        assert fn(4, 128, fake, fake, fake, ctypes.c_void_p((1 << 20) + 2), None) == -1
        assert fn(0, 128, fake, fake, fake, None, None) == 0                 # nothing to do, nothing enqueued
        assert fn(0, 128, None, None, None, None, None) == 0


# --------------------------------------------------------------------------
# host scheduler
# --------------------------------------------------------------------------

def parse_schedule(buf, shape):
    a = buf.numpy().astype(np.int64)
    W, T = int(a[1]), int(a[2])
    workers = a[16:16 + 8 * W].reshape(W, 8)
    tiles = a[16 + 8 * W:16 + 8 * W + 4 * T].reshape(T, 4)
    return dict(hdr=a[:16], W=W, T=T, workers=workers, tiles=tiles)


def pieces_of(sc):
    """Expand worker ranges into (worker, tile, p0, p1, split) pieces."""
    out = []
    for w, (tb, pb, te, pe, fs, *_r) in enumerate(sc["workers"]):
        T = tb
        while T <= te and T < sc["T"]:
            pages = sc["tiles"][T, 0]
            p0 = pb if T == tb else 0
            p1 = pe if T == te else pages
            p1 = min(p1, pages)
            if p0 < p1:
                out.append((w, T, p0, p1, fs if T == tb else 0))
            T += 1
    return out


def check_schedule(seqlens, s_q, h, causal, n_sms):
    b = len(seqlens)
    maxp = max(1, (max(seqlens) + 63) // 64)
    shape = mla.make_shape(b, s_q, h, maxp, 1, causal=causal)
    sc = parse_schedule(mla.mla_plan_schedule_host(shape, torch.tensor(seqlens, dtype=torch.int32), n_sms), shape)
    W = max(1, n_sms // 2)
    tpr = (s_q * h + 127) // 128
    assert sc["W"] == W and sc["T"] == b * tpr
    # visible pages per tile (the rows of a tile are (query token, head) pairs)
    for T in range(b * tpr):
        r, qt = divmod(T, tpr)
        last_row = min(s_q * h, 128 * (qt + 1)) - 1
        i = last_row // h
        L = seqlens[r] - s_q + i + 1 if causal else seqlens[r]
        assert sc["tiles"][T, 0] == (max(L, 0) + 63) // 64
    pcs = pieces_of(sc)
    # every (tile, page) unit exactly once
    cover = {}
    for w, T, p0, p1, split in pcs:
        for p in range(p0, p1):
            assert (T, p) not in cover
            cover[(T, p)] = w
    want = {(T, p) for T in range(b * tpr) for p in range(sc["tiles"][T, 0])}
    assert set(cover) == want
    # split bookkeeping: pieces of a tile are numbered 0..n-1 in order and
    # their slots are disjoint and within 2W
    slots = set()
    by_tile = {}
    for w, T, p0, p1, split in pcs:
        by_tile.setdefault(T, []).append((p0, split))
    for T, lst in by_tile.items():
        n = sc["tiles"][T, 2]
        assert n == len(lst)
        assert [s for _, s in sorted(lst)] == list(range(n))
        if n > 1:
            for k in range(n):
                slot = sc["tiles"][T, 3] + k
                assert slot not in slots
                slots.add(slot)
    assert len(slots) <= 2 * W and sc["hdr"][5] == len(slots)
    for T in range(b * tpr):
        if sc["tiles"][T, 0] == 0:
            assert sc["tiles"][T, 2] == 0
    # balance.  Cut tiles: no worker exceeds the even share by more than one
    # piece's overhead + 1 page.  Whole tiles (chosen when no tile needs
    # cutting): the longest worker is within the split overhead (12 pages) of
    # the even share over the workers that get work.
    cost = np.zeros(W)
    for w, T, p0, p1, split in pcs:
        cost[w] += (p1 - p0) + 2
    total = sc["hdr"][4]
    if (sc["tiles"][:, 2] > 1).any():
        assert cost.max() <= total / W + 2 * 2 + 1
    elif total > 0:
        We = min(W, total)
        assert cost.max() <= -(-total // We) + 12
        assert sc["hdr"][5] == 0 and all(p0 == 0 for _, _, p0, _, _ in pcs)
    return sc


def test_schedule_chooses_whole_tiles_for_similar_lengths():
    """64 requests of 4096 tokens on 74 SM pairs: cutting every tile to the
    even share (57 units) saves less than partials + combine cost, so every
    tile stays whole; the jagged batch is cut."""
    sc = check_schedule([4096] * 64, 1, 128, False, 148)
    assert (sc["tiles"][:, 2] == 1).all() and sc["hdr"][5] == 0
    import mla_workloads as mw
    _, _, _, lens = mw.config_shape(3)
    sc = check_schedule(list(lens), 1, 128, False, 148)
    assert (sc["tiles"][:, 2] > 1).any() and sc["hdr"][5] > 0


@pytest.mark.parametrize("n_sms", [2, 3, 8, 148, 300])
def test_schedule_uniform(n_sms):
    check_schedule([4096] * 64, 1, 128, False, n_sms)


def test_schedule_jagged_and_special_lengths():
    import mla_workloads as mw
    _, _, _, lens = mw.config_shape(3)
    sc = check_schedule(list(lens), 1, 128, False, 148)
    # the forced 131072-token request is cut into several pieces
    r = int(np.argmax(lens))
    assert sc["tiles"][r, 2] > 1
    check_schedule([0, 1, 63, 64, 65, 0, 128, 5000], 1, 16, False, 148)
    check_schedule([0, 0, 0], 1, 128, False, 148)


@pytest.mark.parametrize("lens,n_sms", [([63, 64, 65], 148), ([100, 100], 148), ([256, 256], 148),
                                        ([3000, 64, 1, 2500], 1000), ([1], 4000)])
def test_schedule_more_workers_than_work(lens, n_sms):
    # fewer cost units than workers: the idle workers must not count as pieces
    check_schedule(lens, 1, 128, False, n_sms)
    check_schedule(lens, 1, 16, False, n_sms)


def test_schedule_spec_causal_and_packed_rows():
    check_schedule([4096] * 32, 16, 128, True, 148)
    check_schedule([5, 17, 16, 100], 16, 16, True, 20)   # 2 query tokens per 128-row tile
    check_schedule([3, 200], 4, 48, True, 10)             # tiles straddle query tokens


def test_schedule_clamps_bad_lengths():
    shape = mla.make_shape(3, 1, 128, 2, 1)
    buf = mla.mla_plan_schedule_host(shape, torch.tensor([-5, 1000, 64], dtype=torch.int32), 8)
    sc = parse_schedule(buf, shape)
    assert sc["hdr"][6] != 0                       # status flags the clamp
    assert list(sc["tiles"][:, 0]) == [0, 2, 1]


def test_noalloc_rejects_shapes_beyond_its_static_scratch():
    """mla_decode_fwd_noalloc checks its size limit (16384 tiles) on the host
    before any CUDA call; the pointers are never touched."""
    L = mla.lib()
    fake = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
    for batch, s_q, heads in ((16385, 1, 128), (1, 16385, 128), (8193, 2, 128)):
        shape = mla.make_shape(batch, s_q, heads, 4, 16)
        rc = L.mla_decode_fwd_noalloc(ctypes.byref(shape), fake, fake, None, fake, fake, 0.1, fake, fake, None,
                                      None)
        assert rc == -3, (batch, s_q, heads, rc)
    shape = mla.make_shape(2, 1, 128, 4, 16)
    shape.d_qk = 512
    assert L.mla_decode_fwd_noalloc(ctypes.byref(shape), fake, fake, None, fake, fake, 0.1, fake, fake, None,
                                    None) == -2
    assert L.mla_decode_fwd_noalloc(None, fake, fake, None, fake, fake, 0.1, fake, fake, None, None) == -1
