"""fp64 CPU oracle for MLA decode in absorbed latent space.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code with the CUDA path.

What it computes (page "MLA Cost Analysis & Regime Guide", section
"Absorption Trick"): with the key and value projections absorbed, every head
scores against the shared latent cache directly,

    score  = Qz . Z^T          (Qz = the absorbed 576-d query row, Z = cache rows)
    value  = softmax(score) . Z[:, :512]

which is exactly ordinary softmax attention whose keys are the 576-d cache
rows and whose values are their first 512 entries.  So the oracle is that
plain definition, written out per (request, query token), in float64:

  1. L = t_r - s + i + 1 for query token i of a causal speculative step
     (query i sees keys j <= t_r - s + i); L = t_r otherwise.
  2. C_j = cache row j (j < L) gathered through the block table:
     pool[block_table[r][j // 64], j % 64, :].  For the FP8 cache,
     C_j[:512] = e4m3(byte) * scale_j and C_j[512:] = the bf16 RoPE part.
  3. x_j = softmax_scale * sum_d Q[r, i, h, d] * C_j[d]
  4. lse = m + ln sum_j exp(x_j - m), m = max_j x_j
  5. O[r, i, h, c] = sum_j exp(x_j - lse) * C_j[c], c < 512.

L <= 0 gives O = 0 and lse = -inf.

Token-level sparse decode (the FlashMLA product page lists "token-level
sparse attention" for decoding) takes, per query token (r, i), a list of
cache positions instead of the dense prefix: the plain reading is the same
softmax attention over exactly the listed rows, shared by all heads of that
query token.  Positions outside [0, t_r) (-1 padding) are skipped; a position
listed twice is two keys.

The split form of the same attention for speculative steps ("MLAvar6+
Design" on the same page) keeps the o older tokens in latent form and the n
newest as decompressed per-head keys and values: old token j scores with the
absorbed query against its cache row and contributes its decompressed value
row C_j[:512] . W_kvb2[h]^T; new token m scores with the unabsorbed query
[q_nope | q_pe] against [k_new | its cache row's RoPE part] and contributes
v_new.  One softmax over both.

The two per-head projections on either side of that attention (same page,
"Absorption Trick": the key up-projection is folded into the query, and the
output of the latent attention is decompressed by a separate GEMM) are
written out as their definitions too, with d = 128 head dims and p = 64 RoPE
dims:

  absorb:      Qz[.., j, c] = sum_n q[.., j, n] * Wk[j, c, n]   (c < 512, n < d)
               Qz[.., j, 512 + e] = q[.., j, d + e]             (e < p)
               -- q = [q_nope | q_pe]; head j's keys are K_j = Z . Wk_j
               (Wk_j is 512 x d), so Q . K_j^T = (Q . Wk_j^T) . Z^T.
  decompress:  out[.., j, v] = sum_c O[.., j, c] * Wkvb2[j, v, c]  (v < d)
"""
from __future__ import annotations

import math

import numpy as np
import torch

PAGE = 64
D_QK = 576
D_V = 512
D_HEAD = 128
D_ROPE = 64


# ----------------------------------------------------------------------------
# element decoding
# ----------------------------------------------------------------------------

def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """bf16 -> float64, exact (bf16 is the top half of an IEEE binary32)."""
    bits = t.contiguous().view(torch.int16).numpy().astype(np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def e4m3_table() -> np.ndarray:
    """Value of every e4m3 ("fn" variant: no infinities) byte, from the
    format's definition: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (2^-6 * m/8); S.1111.111 is NaN."""
    tab = np.empty(256, dtype=np.float64)
    for byte in range(256):
        sign = -1.0 if byte & 0x80 else 1.0
        e = (byte >> 3) & 0xF
        m = byte & 0x7
        if e == 0xF and m == 0x7:
            tab[byte] = np.nan
        elif e == 0:
            tab[byte] = sign * math.ldexp(m / 8.0, -6)
        else:
            tab[byte] = sign * math.ldexp(1.0 + m / 8.0, e - 7)
    return tab


_E4M3 = e4m3_table()


def page_rows_f64(pool, page: int, kv_scale=None) -> np.ndarray:
    """One 64-token page as float64 rows [64, 576].

    ``pool`` is bf16 [P, 64, 576], or uint8 [P, 40960] for the FP8 cache whose
    page holds 64x512 e4m3 bytes then 64x64 bf16 RoPE values; the fp32
    per-token scales come in ``kv_scale`` [P, 64]."""
    if pool.dtype == torch.bfloat16:
        return bf16_to_f64(pool[page])
    raw = pool[page].numpy()
    lat = _E4M3[raw[:PAGE * D_V].reshape(PAGE, D_V)]
    sc = kv_scale[page].numpy().astype(np.float64)
    rope = bf16_to_f64(torch.from_numpy(raw[PAGE * D_V:].copy()).view(torch.bfloat16)).reshape(PAGE, D_QK - D_V)
    out = np.empty((PAGE, D_QK), dtype=np.float64)
    out[:, :D_V] = lat * sc[:, None]
    out[:, D_V:] = rope
    return out


def gather_rows(pool, block_table, r: int, n: int, kv_scale=None, start: int = 0) -> np.ndarray:
    """Cache rows start..start+n-1 of request r as float64 [n, 576]."""
    out = np.empty((max(n, 0), D_QK), dtype=np.float64)
    j = start
    while j < start + n:
        pg = int(block_table[r][j // PAGE])
        rows = page_rows_f64(pool, pg, kv_scale)
        lo = j % PAGE
        hi = min(PAGE, lo + (start + n - j))
        out[j - start:j - start + hi - lo] = rows[lo:hi]
        j += hi - lo
    return out


def visible_len(t: int, s_q: int, i: int, causal: bool) -> int:
    """Keys seen by query token i (step 1 of the definition)."""
    return t - s_q + i + 1 if causal else t


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def attend(qrows: np.ndarray, C: np.ndarray, scale: float):
    """Plain softmax attention of query rows [h, 576] over cache rows
    [L, 576] (steps 3-5).  Returns (O [h, 512], lse [h]) in float64."""
    h = qrows.shape[0]
    if C.shape[0] == 0:
        return np.zeros((h, D_V)), np.full(h, -np.inf)
    x = scale * (qrows @ C.T)                       # [h, L]
    m = x.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(x - m).sum(axis=1))
    w = np.exp(x - lse[:, None])
    return w @ C[:, :D_V], lse


def decode(wl, rows=None):
    """Oracle over a whole workload (or over selected (r, i) query tokens).

    ``wl`` carries q bf16 [b, s, h, 576], pool, kv_scale, block_table,
    seqlens, softmax_scale, s_q and causal.  ``rows`` optionally lists
    (r, i) pairs; the result then has shape [len(rows), h, 512] / [len(rows), h].
    Returns (O float64 [b, s, h, 512], lse float64 [b, s, h])."""
    b, s, h, _ = wl.q.shape
    sel = [(r, i) for r in range(b) for i in range(s)] if rows is None else list(rows)
    O = np.zeros((len(sel), h, D_V))
    L = np.zeros((len(sel), h))
    cache = {}
    for n, (r, i) in enumerate(sel):
        t = int(wl.seqlens[r])
        Lv = visible_len(t, s, i, wl.causal)
        if r not in cache:
            cache = {r: gather_rows(wl.pool, wl.block_table, r, t, wl.kv_scale)}
        C = cache[r][:max(Lv, 0)]
        q = bf16_to_f64(wl.q[r, i])
        O[n], L[n] = attend(q, C, wl.softmax_scale)
    if rows is None:
        return O.reshape(b, s, h, D_V), L.reshape(b, s, h)
    return O, L


def sparse_decode(wl, indices: np.ndarray):
    """Token-level sparse decode over the workload's cache.

    indices: int [b, s, k] cache positions per query token; entries outside
    [0, t_r) are skipped.  Returns (O float64 [b, s, h, 512], lse float64
    [b, s, h])."""
    b, s, h, _ = wl.q.shape
    O = np.zeros((b, s, h, D_V))
    L = np.zeros((b, s, h))
    for r in range(b):
        t = int(wl.seqlens[r])
        C_all = gather_rows(wl.pool, wl.block_table, r, t, wl.kv_scale)
        for i in range(s):
            pos = [int(j) for j in indices[r, i] if 0 <= int(j) < t]
            C = C_all[pos] if pos else np.zeros((0, D_QK))
            O[r, i], L[r, i] = attend(bf16_to_f64(wl.q[r, i]), C, wl.softmax_scale)
    return O, L


def decode_chunk(wl, r: int, i: int, start: int, stop: int):
    """Attention of query token (r, i) over its visible keys in [start, stop)
    only: the partial result one split of a split-KV schedule produces."""
    t = int(wl.seqlens[r])
    Lv = visible_len(t, wl.s_q, i, wl.causal)
    stop = min(stop, Lv)
    C = gather_rows(wl.pool, wl.block_table, r, max(stop - start, 0), wl.kv_scale, start=start)
    return attend(bf16_to_f64(wl.q[r, i]), C, wl.softmax_scale)


def combine(parts):
    """Merge partial (O_i, lse_i) results over disjoint key ranges:
    L = ln sum_i e^{lse_i};  O = sum_i e^{lse_i - L} O_i."""
    lses = np.stack([p[1] for p in parts])          # [n, h]
    m = lses.max(axis=0)
    finite = np.isfinite(m)
    msafe = np.where(finite, m, 0.0)
    w = np.exp(lses - msafe)                        # e^{-inf} = 0
    tot = w.sum(axis=0)
    L = np.where(finite, msafe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    O = np.zeros_like(parts[0][0])
    for (Oi, li) in parts:
        wi = np.where(finite, np.exp(li - np.where(finite, L, 0.0)), 0.0)
        O += wi[:, None] * Oi
    return O, L


def brute(wl):
    """Triple loop in pure Python (tiny inputs only): every score, max,
    exponential and weighted sum written out one element at a time, the
    cache read token by token through the block table."""
    b, s, h, _ = wl.q.shape
    O = np.zeros((b, s, h, D_V))
    LSE = np.zeros((b, s, h))
    for r in range(b):
        t = int(wl.seqlens[r])
        for i in range(s):
            Lv = visible_len(t, s, i, wl.causal)
            rows = []
            for j in range(max(Lv, 0)):
                page = int(wl.block_table[r][j // PAGE])
                rows.append(page_rows_f64(wl.pool, page, wl.kv_scale)[j % PAGE].tolist())
            for hh in range(h):
                q = bf16_to_f64(wl.q[r, i, hh]).tolist()
                if not rows:
                    LSE[r, i, hh] = -math.inf
                    continue
                xs = []
                for row in rows:
                    acc = 0.0
                    for d in range(D_QK):
                        acc += q[d] * row[d]
                    xs.append(wl.softmax_scale * acc)
                mx = max(xs)
                z = sum(math.exp(x - mx) for x in xs)
                lse = mx + math.log(z)
                LSE[r, i, hh] = lse
                for c in range(D_V):
                    acc = 0.0
                    for x, row in zip(xs, rows):
                        acc += math.exp(x - lse) * row[c]
                    O[r, i, hh, c] = acc
    return O, LSE


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), returned as
    float64: the comparison target for bf16 kernel outputs."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                               # x = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                          # below 2^-126: fixed subnormal spacing
    ulp = np.ldexp(1.0, e - 8)                       # 8 significant bits
    with np.errstate(invalid="ignore", over="ignore"):
        r = np.round(x / ulp) * ulp                  # np.round: ties to even
        r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, x), r)
    return np.where(np.isfinite(x), r, x)


# ----------------------------------------------------------------------------
# projections on either side of the latent attention
# ----------------------------------------------------------------------------

def absorb(q: np.ndarray, w_k: np.ndarray) -> np.ndarray:
    """Absorbed query rows (page "MLA Cost Analysis & Regime Guide",
    "Absorption Trick": Q . K^T = (Q . Wk^T) . Z^T).

    q    float64 [..., h, d + p] = [q_nope | q_pe]
    w_k  float64 [h, 512, d]: head j's keys are K_j = Z . w_k[j]
    Returns float64 [..., h, 576] = [q_nope . w_k[j]^T | q_pe]."""
    lat = np.einsum("...jn,jcn->...jc", q[..., :D_HEAD], w_k)
    return np.concatenate([lat, q[..., D_HEAD:D_HEAD + D_ROPE]], axis=-1)


def decompress(o_lat: np.ndarray, w_kvb2: np.ndarray) -> np.ndarray:
    """Per-head output of the latent attention mapped back to head space
    (same page and section: O_latent . W_kvb2^T, run after the attention).

    o_lat   float64 [..., h, 512]
    w_kvb2  float64 [h, d, 512]: head j's values are V_j = Z . w_kvb2[j]^T
    Returns float64 [..., h, d]."""
    return np.einsum("...jc,jvc->...jv", o_lat, w_kvb2)


def new_token_attention(wl, q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, n_new: int):
    """Attention of every query row over the n decompressed newest tokens
    alone (the second part of the split form): keys [k_new | the cache
    row's RoPE part], values v_new, the same positions and visibility as
    mlavar6_decode.  Returns (o [b, s, h, d], lse [b, s, h]); a row that
    sees none of them gives o = 0, lse = -inf."""
    b, s, h, _ = q.shape
    d = D_HEAD
    out = np.zeros((b, s, h, d))
    lse = np.full((b, s, h), -np.inf)
    for r in range(b):
        t = int(wl.seqlens[r])
        C = gather_rows(wl.pool, wl.block_table, r, t, wl.kv_scale)
        for i in range(s):
            Lv = max(visible_len(t, s, i, wl.causal), 0)
            ms = np.arange(n_new)
            pos = t - n_new + ms
            keep = (pos >= 0) & (pos < Lv)
            ms, pos = ms[keep], pos[keep]
            if ms.size == 0:
                continue
            for hh in range(h):
                x = wl.softmax_scale * (k_new[r, ms, hh] @ q[r, i, hh, :d] + C[pos, D_V:] @ q[r, i, hh, d:])
                m = x.max()
                lse[r, i, hh] = m + math.log(np.exp(x - m).sum())
                out[r, i, hh] = np.exp(x - lse[r, i, hh]) @ v_new[r, ms, hh]
    return out, lse


def mlavar6_decode(wl, qz: np.ndarray, q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray,
                   w_kvb2: np.ndarray, n_new: int, rows=None):
    """Split latent + decompressed attention (page "MLA Cost Analysis &
    Regime Guide", "MLAvar6+ Design"), in float64.

    wl      the workload: cache pool, block table, seqlens, softmax_scale,
            s_q, causal (its q is not used)
    qz      [b, s, h, 576] absorbed query (old tokens)
    q       [b, s, h, d + p] unabsorbed query [q_nope | q_pe] (new tokens)
    k_new   [b, n, h, d] decompressed keys of each request's n newest tokens
    v_new   [b, n, h, d] their decompressed values
    w_kvb2  [h, d, 512] value decompression of the old tokens
    Token positions: old j < t - n, new m at position t - n + m (m with a
    negative position, when t < n, does not exist); query i sees positions
    below visible_len(t, s, i, causal).
    ``rows`` optionally lists (r, i) query tokens; the result then has shape
    [len(rows), h, d] / [len(rows), h].
    Returns (out [b, s, h, d], lse [b, s, h])."""
    b, s, h, _ = qz.shape
    d = D_HEAD
    sel = [(r, i) for r in range(b) for i in range(s)] if rows is None else list(rows)
    out = np.zeros((len(sel), h, d))
    lse = np.zeros((len(sel), h))
    C, C_r = None, -1
    for n_sel, (r, i) in enumerate(sel):
        t = int(wl.seqlens[r])
        if r != C_r:
            C, C_r = gather_rows(wl.pool, wl.block_table, r, t, wl.kv_scale), r
        o = max(t - n_new, 0)
        Lv = max(visible_len(t, s, i, wl.causal), 0)
        jo = min(o, Lv)                                   # visible old tokens
        ms = np.arange(n_new)
        pos = t - n_new + ms
        keep = (pos >= 0) & (pos < Lv)                    # visible new tokens
        ms, pos = ms[keep], pos[keep]
        for hh in range(h):
            x_old = wl.softmax_scale * (C[:jo] @ qz[r, i, hh])
            x_new = wl.softmax_scale * (k_new[r, ms, hh] @ q[r, i, hh, :d] + C[pos, D_V:] @ q[r, i, hh, d:])
            x = np.concatenate([x_old, x_new])
            if x.size == 0:
                lse[n_sel, hh] = -np.inf
                continue
            m = x.max()
            z = np.exp(x - m).sum()
            lse[n_sel, hh] = m + math.log(z)
            w = np.exp(x - lse[n_sel, hh])
            vals = np.concatenate([C[:jo, :D_V] @ w_kvb2[hh].T, v_new[r, ms, hh]])
            out[n_sel, hh] = w @ vals
    if rows is None:
        return out.reshape(b, s, h, d), lse.reshape(b, s, h)
    return out, lse
