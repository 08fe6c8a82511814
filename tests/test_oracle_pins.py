"""Pins for the fp64 oracle: each check ties it to something other than itself
(values printed on the pages, closed forms, a library routine, brute force).

Citations name the "MLA Cost Analysis & Regime Guide" page (sections "Cost
Models", "Absorption Trick", "Tensor Shapes", "Historical Baselines") and the
FlashMLA-2 newsletter page (section "Architectural Analysis": split-KV
balancing across SMs).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_decode as om
import mla_workloads as mw
from mla_workloads import cost
from conftest import load_golden

SCALE = 1.0 / math.sqrt(192.0)


# --------------------------------------------------------------------------
# cost model vs the numbers the page prints ("Cost Models")
# --------------------------------------------------------------------------

def test_cost_model_matches_printed_values():
    g = load_golden("cost_model.txt")
    b, h, t, k, p, d = 64, 128, 4096, 512, 64, 128
    ai = cost.mla_flops(b, h, 1, t) / cost.mla_bytes(b, h, 1, t)
    assert abs(ai - g["flashmla_ai_s1"][0]) <= g["flashmla_ai_s1"][1]
    fa1 = cost.fa_flops(b, h, 1, t) / cost.fa_bytes(b, h, 1, t)
    assert abs(fa1 - g["fa_ai_s1"][0]) <= g["fa_ai_s1"][1]
    fa1024 = cost.fa_flops(b, h, 1024, t) / cost.fa_bytes(b, h, 1024, t)
    assert abs(fa1024 - g["fa_ai_s1024"][0]) <= g["fa_ai_s1024"][1]
    # per-token FLOP factors 2k+p and 2d+p, and their ratio
    assert cost.mla_flops(1, 1, 1, 1) / 2 == g["flashmla_flop_factor"][0]
    assert cost.fa_flops(1, 1, 1, 1) / 2 == g["fa_flop_factor"][0]
    ratio = cost.mla_flops(b, h, 1, t) / cost.fa_flops(b, h, 1, t)
    assert abs(ratio - g["flops_per_token_ratio"][0]) <= g["flops_per_token_ratio"][1]
    # the recomputed value the roofline uses (no rounding): 228.30
    assert abs(ai - 228.30) < 0.01


def test_cost_model_batch_independence_and_jagged_sum():
    # AI at s=1 does not depend on b; a jagged batch sums its lengths
    a1 = cost.mla_flops(1, 128, 1, 4096) / cost.mla_bytes(1, 128, 1, 4096)
    a2 = cost.mla_flops(64, 128, 1, 4096) / cost.mla_bytes(64, 128, 1, 4096)
    assert abs(a1 - a2) < 1e-9
    assert cost.mla_flops(3, 128, 1, None, sum_t=100 + 200 + 300) == cost.mla_flops(3, 128, 1, 200)


def test_mlavar6_flops_interpolate_between_the_two_models():
    # the split-cache design reduces to the latent model at n=0 and to the
    # decompressed model at o=0 ("MLAvar6+ Design")
    b, h, s, t = 32, 128, 16, 4096
    assert cost.mlavar6_flops(b, h, s, t, 0) == cost.mla_flops(b, h, s, t)
    assert cost.mlavar6_flops(b, h, s, 0, t) == cost.fa_flops(b, h, s, t)


def test_latency_table_ratios():
    g = load_golden("rtx5090_latency_table.txt")
    sp = g["fa_s1_us"][0] / g["flashmla_s1_us"][0]
    assert abs(sp - g["decode_speedup_vs_fa"][0]) <= g["decode_speedup_vs_fa"][1]
    gain = 100.0 * (g["flashmla_s16_us"][0] - g["mlavar6_v3_s16_us"][0]) / g["flashmla_s16_us"][0]
    assert abs(gain - g["mlavar6_gain_s16_pct"][0]) <= g["mlavar6_gain_s16_pct"][1]


# --------------------------------------------------------------------------
# element decoding vs library conversions
# --------------------------------------------------------------------------

def test_e4m3_table_matches_torch():
    tab = om.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(tab))
    assert np.array_equal(tab[~nan], ref[~nan])
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(4096, generator=g) * 100).to(torch.bfloat16)
    x[:4] = torch.tensor([0.0, -0.0, 1e-40, -3e38]).to(torch.bfloat16)
    assert np.array_equal(om.bf16_to_f64(x), x.to(torch.float64).numpy())


def test_round_bf16_matches_torch_rne():
    g = torch.Generator().manual_seed(2)
    f = torch.randn(100000, generator=g, dtype=torch.float32) * 3
    f[:3] = torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)])  # exact ties
    ref = f.to(torch.bfloat16).to(torch.float64).numpy()
    got = om.round_bf16(f.to(torch.float64).numpy())
    assert np.array_equal(ref, got)


# --------------------------------------------------------------------------
# attention: brute force, closed forms, library routine
# --------------------------------------------------------------------------

def _tiny(seqlens, h=4, s_q=1, causal=False, cache_dtype="bf16", seed=3, contiguous=False):
    return mw.make(len(seqlens), s_q, h, list(seqlens), causal=causal, cache_dtype=cache_dtype,
                   seed=seed, contiguous=contiguous)


@pytest.mark.parametrize("lens", [[1], [63], [64], [65], [1, 130, 64]])
def test_vectorised_matches_brute_force(lens):
    wl = _tiny(lens, h=3)
    O, L = oracle.decode(wl)
    Ob, Lb = oracle.brute(wl)
    assert np.max(np.abs(O - Ob)) < 1e-12
    assert np.max(np.abs(L - Lb)) < 1e-12


def test_brute_force_causal_and_fp8():
    wl = _tiny([70, 5], h=2, s_q=3, causal=True)
    O, L = oracle.decode(wl)
    Ob, Lb = oracle.brute(wl)
    assert np.max(np.abs(O - Ob)) < 1e-12 and np.max(np.abs(L - Lb)) < 1e-12
    wl8 = _tiny([67], h=2, cache_dtype="fp8")
    O, L = oracle.decode(wl8)
    Ob, Lb = oracle.brute(wl8)
    assert np.max(np.abs(O - Ob)) < 1e-12 and np.max(np.abs(L - Lb)) < 1e-12


def test_brute_force_config1_shape():
    # the tiny workload's exact shape (b=2, h=16, t=256, contiguous), two heads
    # checked by brute force to keep the pure-Python loop short
    wl = mw.make_config(1)
    O, L = oracle.decode(wl)
    sub = mw.make(2, 1, 16, 256, contiguous=True, seed=0)
    sub.q = sub.q[:, :, :2].contiguous()
    Ob, Lb = oracle.brute(sub)
    assert np.max(np.abs(O[:, :, :2] - Ob)) < 1e-12 and np.max(np.abs(L[:, :, :2] - Lb)) < 1e-12


def _absorption_case(seed=0, t=96, h=4):
    """Random DeepSeek-style factors: per head W_k, W_v (k x d), q_nope (d),
    q_pe (p); a latent cache Z (t x k) and RoPE keys KPE (t x p)."""
    g = torch.Generator().manual_seed(seed)
    k, d, p = 512, 128, 64
    Wk = torch.randn(h, k, d, generator=g, dtype=torch.float64) / math.sqrt(k)
    Wv = torch.randn(h, k, d, generator=g, dtype=torch.float64) / math.sqrt(k)
    qn = torch.randn(h, d, generator=g, dtype=torch.float64)
    qp = torch.randn(h, p, generator=g, dtype=torch.float64)
    Z = torch.randn(t, k, generator=g, dtype=torch.float64)
    KPE = torch.randn(t, p, generator=g, dtype=torch.float64)
    return Wk, Wv, qn, qp, Z, KPE


def _mha_reference(Wk, Wv, qn, qp, Z, KPE):
    """Ordinary multi-head attention with decompressed per-head keys
    K_h = [Z Wk_h | KPE] and values V_h = Z Wv_h, through the library's
    scaled_dot_product_attention in float64, scale 1/sqrt(d + p)."""
    h = Wk.shape[0]
    K = torch.stack([torch.cat([Z @ Wk[i], KPE], dim=1) for i in range(h)])      # h, t, 192
    V = torch.stack([Z @ Wv[i] for i in range(h)])                               # h, t, 128
    Q = torch.cat([qn, qp], dim=1)[:, None, :]                                   # h, 1, 192
    return torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=SCALE)[:, 0]


def _latent_path(attend, Wk, Wv, qn, qp, Z, KPE):
    """Absorbed path: Qz_h = [Wk_h qn_h | qp_h], cache rows [Z | KPE], the
    oracle's attention, then decompression O_lat,h Wv_h."""
    h = Wk.shape[0]
    Qz = torch.stack([torch.cat([Wk[i] @ qn[i], qp[i]]) for i in range(h)]).numpy()
    C = torch.cat([Z, KPE], dim=1).numpy()
    Olat, _ = attend(Qz, C, SCALE)
    return np.stack([Olat[i] @ Wv[i].numpy() for i in range(h)])


def test_absorption_identity():
    case = _absorption_case()
    ref = _mha_reference(*case).numpy()
    got = _latent_path(oracle.attend, *case)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_absorb_and_decompress_reach_plain_mha():
    # the oracle's projections around its attention give the same heads as
    # ordinary MHA over decompressed keys and values: q = [q_nope | q_pe],
    # Wk_h is 512 x d (K_h = Z Wk_h), W_kvb2_h = Wv_h^T is d x 512
    Wk, Wv, qn, qp, Z, KPE = case = _absorption_case(seed=3, t=130, h=5)
    ref = _mha_reference(*case).numpy()
    q = torch.cat([qn, qp], dim=1).numpy()                       # h, 192
    qz = oracle.absorb(q, Wk.numpy())                            # h, 576
    C = torch.cat([Z, KPE], dim=1).numpy()
    olat, _ = oracle.attend(qz, C, SCALE)
    got = oracle.decompress(olat, Wv.transpose(1, 2).numpy())
    assert got.shape == ref.shape == (5, 128)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_projections_on_selector_weights():
    # closed forms: a weight that selects one input column per output column,
    # scaled differently per head, must route exactly those values
    g = torch.Generator().manual_seed(11)
    R, h = 3, 4
    q = torch.randn(R, h, 192, generator=g, dtype=torch.float64).numpy()
    wk = np.zeros((h, 512, 128))
    for j in range(h):
        for n in range(128):
            wk[j, (n + 100 * j) % 512, n] = j + 1.0              # latent c <- (j+1) q_nope[n]
    qz = oracle.absorb(q, wk)
    want = np.zeros((R, h, 576))
    for j in range(h):
        for n in range(128):
            want[:, j, (n + 100 * j) % 512] = (j + 1.0) * q[:, j, n]
    want[..., 512:] = q[..., 128:]
    assert np.array_equal(qz, want)
    o = torch.randn(R, h, 512, generator=g, dtype=torch.float64).numpy()
    wv = np.zeros((h, 128, 512))
    for j in range(h):
        for v in range(128):
            wv[j, v, (3 * v + 128 * j) % 512] = -(j + 2.0)
    out = oracle.decompress(o, wv)
    for j in range(h):
        for v in range(128):
            assert np.array_equal(out[:, j, v], -(j + 2.0) * o[:, j, (3 * v + 128 * j) % 512])


# ---- token-level sparse decode ---------------------------------------------

def _rows_as_workload(wl, r, i, pos):
    """A one-request workload whose contiguous cache holds exactly the bf16
    rows at positions `pos` of request r, in that order, queried by (r, i)."""
    n = len(pos)
    pages = max(1, (n + 63) // 64)
    pool = torch.zeros((pages, 64, 576), dtype=torch.bfloat16)
    for k, j in enumerate(pos):
        pool[k // 64, k % 64] = wl.pool[int(wl.block_table[r][j // 64]), j % 64]
    return mw.Workload(name="rows", batch=1, s_q=1, num_heads=wl.num_heads, causal=False, cache_dtype="bf16",
                       seqlens=np.array([n], dtype=np.int32),
                       block_table=np.arange(pages, dtype=np.int32)[None, :], q=wl.q[r:r + 1, i:i + 1].clone(),
                       pool=pool, kv_scale=None, softmax_scale=wl.softmax_scale)


@pytest.mark.parametrize("cache_dtype", ["bf16", "fp8"])
def test_sparse_with_every_position_is_the_dense_decode(cache_dtype):
    wl = _tiny([70, 130, 5], h=3, s_q=2, cache_dtype=cache_dtype)
    idx = np.full((3, 2, 140), -1, dtype=np.int32)
    for r, t in enumerate(wl.seqlens):
        idx[r, :, :t] = np.arange(t)
    O, L = oracle.sparse_decode(wl, idx)
    Od, Ld = oracle.decode(wl)
    assert np.max(np.abs(O - Od)) < 1e-12 and np.max(np.abs(L - Ld)) < 1e-12


def test_sparse_matches_brute_force_on_the_selected_rows():
    # the rows are found through the block table: a brute-force triple loop over
    # a contiguous copy of exactly those rows must agree
    wl = _tiny([150, 90], h=2, s_q=2, seed=8)
    rng = np.random.default_rng(1)
    idx = np.full((2, 2, 12), -1, dtype=np.int32)
    for r, t in enumerate(wl.seqlens):
        for i in range(2):
            idx[r, i, :10] = rng.choice(int(t), size=10, replace=False)
    idx[0, 1, 10] = 149          # the last position
    idx[1, 0, 11] = 90           # one past the end: skipped
    O, L = oracle.sparse_decode(wl, idx)
    for r in range(2):
        for i in range(2):
            pos = [int(j) for j in idx[r, i] if 0 <= j < wl.seqlens[r]]
            Ob, Lb = oracle.brute(_rows_as_workload(wl, r, i, pos))
            assert np.max(np.abs(O[r, i] - Ob[0, 0])) < 1e-12
            assert np.max(np.abs(L[r, i] - Lb[0, 0])) < 1e-12


def test_sparse_order_padding_and_duplicates():
    wl = _tiny([200], h=4, seed=9)
    rng = np.random.default_rng(2)
    sel = rng.choice(200, size=37, replace=False).astype(np.int32)
    a = sel[None, None, :]
    b = np.concatenate([rng.permutation(sel), [-1, -1, 200, 1000]]).astype(np.int32)[None, None, :]
    Oa, La = oracle.sparse_decode(wl, a)
    Ob, Lb = oracle.sparse_decode(wl, b)
    assert np.max(np.abs(Oa - Ob)) < 1e-12 and np.max(np.abs(La - Lb)) < 1e-12     # order, padding
    # a position listed twice is two keys: with keys {u, v} and u twice the
    # weights are 2e^{x_u} : e^{x_v}
    u, v = int(sel[0]), int(sel[1])
    Od, Ld = oracle.sparse_decode(wl, np.array([[[u, v, u]]], dtype=np.int32))
    C = om.gather_rows(wl.pool, wl.block_table, 0, 200)
    q = om.bf16_to_f64(wl.q[0, 0])
    xu, xv = SCALE * (q @ C[u]), SCALE * (q @ C[v])
    wu = 2 * np.exp(xu) / (2 * np.exp(xu) + np.exp(xv))
    want = wu[:, None] * C[u, :512] + (1 - wu)[:, None] * C[v, :512]
    assert np.max(np.abs(Od[0, 0] - want)) < 1e-12
    assert np.max(np.abs(Ld[0, 0] - np.log(2 * np.exp(xu) + np.exp(xv)))) < 1e-12
    # nothing valid: O = 0, lse = -inf
    Oz, Lz = oracle.sparse_decode(wl, np.array([[[-1, 200, -7]]], dtype=np.int32))
    assert np.all(Oz == 0) and np.all(np.isneginf(Lz))


# ---- MLAvar6+: old tokens in latent form, the n newest decompressed ---------

def _var6_case(n_new, seed=5, cache_dtype="bf16"):
    """A causal speculative batch, random per-head projections, and the
    exact (fp64) decompression of each request's n newest tokens; slots of
    positions that do not exist (t < n) are NaN."""
    wl = _tiny([150, 70], h=3, s_q=3, causal=True, seed=seed, cache_dtype=cache_dtype)
    g = torch.Generator().manual_seed(seed + 1)
    h = wl.num_heads
    wk = (torch.randn(h, 512, 128, generator=g, dtype=torch.float64) / math.sqrt(512)).numpy()
    wv = (torch.randn(h, 128, 512, generator=g, dtype=torch.float64) / math.sqrt(512)).numpy()
    q = torch.randn(wl.batch, wl.s_q, h, 192, generator=g, dtype=torch.float64).numpy()
    qz = oracle.absorb(q, wk)
    k_new = np.full((wl.batch, n_new, h, 128), np.nan)
    v_new = np.full((wl.batch, n_new, h, 128), np.nan)
    for r, t in enumerate(wl.seqlens):
        C = om.gather_rows(wl.pool, wl.block_table, r, int(t), wl.kv_scale)
        for m in range(n_new):
            p = int(t) - n_new + m
            if p >= 0:
                k_new[r, m] = np.einsum("c,jcn->jn", C[p, :512], wk)
                v_new[r, m] = np.einsum("c,jvc->jv", C[p, :512], wv)
    return wl, wk, wv, q, qz, k_new, v_new


@pytest.mark.parametrize("n_new,cache_dtype", [(0, "bf16"), (1, "bf16"), (3, "bf16"), (64, "bf16"),
                                               (100, "bf16"), (150, "bf16"), (64, "fp8")])
def test_mlavar6_with_exact_decompression_is_the_latent_path(n_new, cache_dtype):
    # whatever n, keeping the newest tokens decompressed changes nothing when
    # their keys and values are the exact projections of their latent rows;
    # n = 100 > t = 70 for the second request, n = 150 = t makes the first
    # request fully decompressed (ordinary MHA)
    wl, wk, wv, q, qz, k_new, v_new = _var6_case(n_new, cache_dtype=cache_dtype)
    out, lse = oracle.mlavar6_decode(wl, qz, q, k_new, v_new, wv, n_new)
    for r, t in enumerate(wl.seqlens):
        C = om.gather_rows(wl.pool, wl.block_table, r, int(t), wl.kv_scale)
        for i in range(wl.s_q):
            L = om.visible_len(int(t), wl.s_q, i, True)
            olat, lref = oracle.attend(qz[r, i], C[:L], wl.softmax_scale)
            assert np.max(np.abs(out[r, i] - oracle.decompress(olat, wv))) < 1e-12
            assert np.max(np.abs(lse[r, i] - lref)) < 1e-12


@pytest.mark.parametrize("n_new", [3, 64, 100])
def test_mlavar6_is_the_merge_of_its_two_parts(n_new):
    # the joint softmax over old and new tokens equals the log-sum-exp merge
    # of the decompressed latent attention over the old tokens and the
    # attention over the new ones (arbitrary k_new / v_new: the identity
    # does not depend on them being projections)
    wl, wk, wv, q, qz, _, _ = _var6_case(n_new, seed=9)
    g = np.random.default_rng(3)
    k_new = g.standard_normal((wl.batch, n_new, wl.num_heads, 128))
    v_new = g.standard_normal((wl.batch, n_new, wl.num_heads, 128))
    out, lse = oracle.mlavar6_decode(wl, qz, q, k_new, v_new, wv, n_new)
    o_new, l_new = oracle.new_token_attention(wl, q, k_new, v_new, n_new)
    for r, t in enumerate(wl.seqlens):
        C = om.gather_rows(wl.pool, wl.block_table, r, int(t), wl.kv_scale)
        old = max(int(t) - n_new, 0)
        for i in range(wl.s_q):
            olat, l_old = oracle.attend(qz[r, i], C[:old], wl.softmax_scale)
            o, L = oracle.combine([(oracle.decompress(olat, wv), l_old), (o_new[r, i], l_new[r, i])])
            assert np.max(np.abs(out[r, i] - o)) < 1e-12 and np.max(np.abs(lse[r, i] - L)) < 1e-12


def test_uniform_scores_give_mean_of_values():
    # Q = 0: every score is 0, so the weights are 1/L, O is the mean of the
    # value rows and lse = ln L
    wl = _tiny([1, 77, 200], h=2)
    wl.q.zero_()
    O, L = oracle.decode(wl)
    for r, t in enumerate(wl.seqlens):
        C = om.gather_rows(wl.pool, wl.block_table, r, int(t))
        assert np.max(np.abs(O[r, 0] - C[:, :512].mean(axis=0))) < 1e-12
        assert np.max(np.abs(L[r, 0] - math.log(t))) < 1e-12


def test_rows_sum_to_one():
    # a latent column that is 1 in every cache row must come out as exactly 1
    wl = _tiny([150, 3], h=4)
    wl.pool[:, :, 17] = 1.0
    O, _ = oracle.decode(wl)
    assert np.max(np.abs(O[..., 17] - 1.0)) < 1e-12


def test_single_key_returns_its_value():
    wl = _tiny([1], h=4)
    O, L = oracle.decode(wl)
    C = om.gather_rows(wl.pool, wl.block_table, 0, 1)
    q = om.bf16_to_f64(wl.q[0, 0])
    assert np.array_equal(O[0, 0], np.broadcast_to(C[0, :512], (4, 512)))
    assert np.max(np.abs(L[0, 0] - SCALE * (q @ C[0]))) < 1e-12


def test_zero_length_request():
    wl = _tiny([0, 10], h=2)
    O, L = oracle.decode(wl)
    assert np.all(O[0] == 0) and np.all(np.isneginf(L[0]))


@pytest.mark.parametrize("cuts", [[], [64], [1, 2, 3], [63, 64, 65, 300], list(range(64, 640, 64))])
def test_split_combine_equals_unsplit(cuts):
    # the split-KV merge (each piece's lse-weighted partial) reproduces the
    # unsplit result: FlashMLA-2 newsletter, "Architectural Analysis"
    wl = _tiny([700], h=3)
    O, L = oracle.decode(wl)
    edges = [0] + cuts + [700]
    parts = [oracle.decode_chunk(wl, 0, 0, a, b) for a, b in zip(edges[:-1], edges[1:])]
    Oc, Lc = oracle.combine(parts)
    assert np.max(np.abs(Oc - O[0, 0])) < 1e-12 and np.max(np.abs(Lc - L[0, 0])) < 1e-12


def test_causal_matches_masked_sdpa():
    # the speculative step: query i sees keys j <= t - s + i; checked against
    # the library attention with an explicit boolean mask
    wl = _tiny([100, 64], h=3, s_q=5, causal=True)
    O, L = oracle.decode(wl)
    for r, t in enumerate(wl.seqlens):
        t = int(t)
        C = torch.from_numpy(om.gather_rows(wl.pool, wl.block_table, r, t))
        Q = torch.from_numpy(om.bf16_to_f64(wl.q[r])).permute(1, 0, 2)          # h, s, 576
        mask = torch.arange(t)[None, :] <= (t - 5 + torch.arange(5))[:, None]     # s, t
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, C[None].expand(3, t, 576), C[None, :, :512].expand(3, t, 512), attn_mask=mask, scale=SCALE)
        assert np.max(np.abs(O[r] - ref.permute(1, 0, 2).numpy())) < 1e-12


def test_fp8_pages_dequantise_like_torch():
    wl = _tiny([130], h=1, cache_dtype="fp8")
    for pg in range(wl.num_pages):
        rows = om.page_rows_f64(wl.pool, pg, wl.kv_scale)
        raw = wl.pool[pg]
        lat = raw[:64 * 512].view(torch.float8_e4m3fn).to(torch.float64).reshape(64, 512)
        lat = lat * wl.kv_scale[pg].to(torch.float64)[:, None]
        rope = raw[64 * 512:].view(torch.bfloat16).to(torch.float64).reshape(64, 64)
        assert np.array_equal(rows[:, :512], lat.numpy())
        assert np.array_equal(rows[:, 512:], rope.numpy())


def test_nan_in_unused_slots_is_ignored():
    wl = _tiny([70, 10], h=2)
    O, L = oracle.decode(wl)
    # poison every slot past each request's length and every unreferenced page
    used = set()
    for r, t in enumerate(wl.seqlens):
        n = (int(t) + 63) // 64
        used |= set(int(x) for x in wl.block_table[r, :n])
        last = int(wl.block_table[r, n - 1])
        if t % 64:
            wl.pool[last, int(t) % 64:] = float("nan")
    extra = mw.make(1, 1, 1, [64], seed=9).pool.fill_(float("nan"))
    wl.pool = torch.cat([wl.pool, extra])
    O2, L2 = oracle.decode(wl)
    assert np.isfinite(O2).all() and np.array_equal(O, O2) and np.array_equal(L, L2)


# --------------------------------------------------------------------------
# planted mistakes: each must trip at least one pin above
# --------------------------------------------------------------------------

def _attend_no_rope(qrows, C, scale):
    return om.attend(np.concatenate([qrows[:, :512], np.zeros_like(qrows[:, 512:])], 1), C, scale)


def _attend_wrong_scale(qrows, C, scale):
    return om.attend(qrows, C, 1.0 / math.sqrt(576.0))


def _attend_values_from_tail(qrows, C, scale):
    O, L = om.attend(qrows, C, scale)
    x = scale * (qrows @ C.T)
    w = np.exp(x - L[:, None])
    return w @ C[:, 64:], L


def _attend_transposed(qrows, C, scale):
    O, L = om.attend(qrows, C, scale)
    return O[:, ::-1].copy(), L


@pytest.mark.parametrize("bad", [_attend_no_rope, _attend_wrong_scale, _attend_values_from_tail,
                                 _attend_transposed])
def test_planted_mistakes_are_caught(bad):
    case = _absorption_case(seed=5)
    ref = _mha_reference(*case).numpy()
    got = _latent_path(bad, *case)
    assert np.max(np.abs(got - ref)) > 1e-3


def test_planted_page_index_mistake_is_caught(monkeypatch):
    # a wrong block-table lookup in the vectorised oracle must disagree with
    # the brute-force loop, which reads the table on its own
    wl = _tiny([130], h=2)
    Ob, _ = oracle.brute(wl)
    orig = om.gather_rows

    def wrong_page(pool, table, r, n, kv_scale=None, start=0):
        return orig(pool, np.roll(np.asarray(table), 1, axis=1), r, n, kv_scale, start)
    monkeypatch.setattr(om, "gather_rows", wrong_page)
    O2, _ = om.decode(wl)
    assert np.max(np.abs(O2 - Ob)) > 1e-3
