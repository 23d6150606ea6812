"""CPU oracle for absorbed-MLA decode: plain, slow, fp64.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline / reference arm may import this module; the library never does,
and it shares no code with the CUDA path (the only common input is the seeded
generator, which holds none of this arithmetic).

What it computes, and where each step is defined:

* Latent projection  c_t = W^DKV h_t                      -- "MLA deep compression"
  (operatorworld.com), section on the low-rank projection (first equation).
* Per-head up-projection  k^C_{t,i} = W^UK_i c_t,  v_{t,i} = W^UV_i c_t
  -- same page and section, second equation.  The page prints the key matrix
  as W^KR_i there; this oracle reads it as W^UK_i (the content-key
  up-projection), because the same page later reserves W^KR for the RoPE key
  projection from h, and "Attention-head anatomy" §5 names W^UK as the matrix
  folded into the query path.
* Decoupled RoPE  k^R_t = RoPE(W^KR h_t) shared by all heads,
  q^R_i = RoPE(W^QR_i h), score = content dot product + RoPE dot product
  -- "MLA deep compression", section on decoupled RoPE; "Attention-head
  anatomy" §5 ("add the two dot products").  The pages give no RoPE
  convention; this oracle uses rotations of consecutive pairs (2k, 2k+1) by
  angle pos * base^(-2k/d_R).
* Softmax over cached positions, o_i = sum_j a_ij v_{j,i}  -- "MLA deep
  compression", section on absorption, output-side equation.
* Absorption (for the separate absorbed helper and for checking the GPU's
  intermediate u): W^QK_i = (W^UK_i)^T W^Q_i, score = (W^QK_i h)^T c,
  u_i = sum_j a_ij c_j, o_i = W^UV_i u_i -- same section, both equations.
* Cache width d_c + d_R and the KV-bytes formula 2*layers*kv_heads*head_dim*
  bytes -- "MLA deep compression", decoupled-RoPE section; "Attention-head
  anatomy" §2 and §4.

Readings where the pages are silent: the softmax scale is a parameter; the
s_q query rows of a sequence of length L sit at positions L - s_q + r and row
r sees cached positions j <= L - s_q + r; lse is the natural log of
sum_j exp(scale * s_j).

Every function here is pinned by tests/test_oracle.py against brute force,
closed forms and the figures the pages print.
"""
from __future__ import annotations

import math

import numpy as np

f64 = np.float64


# ----------------------------------------------------------------------------
# closed-form cache arithmetic
# ----------------------------------------------------------------------------
def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_elem: int) -> int:
    """Per-token K/V cache bytes: 2 * layers * kv_heads * head_dim * bytes
    ("Attention-head anatomy" §2, the one formula)."""
    return 2 * layers * kv_heads * head_dim * bytes_per_elem


def mla_cache_elems(d_c: int, d_R: int) -> int:
    """Cached values per token per layer under MLA: the latent plus the shared
    RoPE key ("MLA deep compression", decoupled-RoPE section)."""
    return d_c + d_R


def mha_kv_elems(n_h: int, d_h: int) -> int:
    """K and V values per token per layer when every head caches its own pair
    ("MLA deep compression", opening paragraph)."""
    return 2 * n_h * d_h


# ----------------------------------------------------------------------------
# projections
# ----------------------------------------------------------------------------
def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate consecutive pairs (2k, 2k+1) of the last axis of x by angle
    pos * base^(-2k/d).  ``pos`` broadcasts against x[..., 0]."""
    x = np.asarray(x, dtype=f64)
    d = x.shape[-1]
    assert d % 2 == 0
    k = np.arange(d // 2, dtype=f64)
    theta = np.power(f64(base), -2.0 * k / d)                    # [d/2]
    ang = np.asarray(pos, dtype=f64)[..., None] * theta           # [..., d/2]
    cos, sin = np.cos(ang), np.sin(ang)
    even, odd = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = even * cos - odd * sin
    out[..., 1::2] = even * sin + odd * cos
    return out


def latent(W_DKV: np.ndarray, h: np.ndarray) -> np.ndarray:
    """c = W^DKV h for every row of h: [..., d_model] -> [..., d_c]."""
    return np.asarray(h, f64) @ np.asarray(W_DKV, f64).T


def rope_key(W_KR: np.ndarray, h: np.ndarray, pos, base: float) -> np.ndarray:
    """k^R = RoPE(W^KR h, pos): [..., d_model] -> [..., d_R]."""
    return rope(np.asarray(h, f64) @ np.asarray(W_KR, f64).T, pos, base)


def query_head(W_Q_i, W_QR_i, h, pos, base):
    """Non-absorbed query of head i: [W^Q_i h || RoPE(W^QR_i h, pos)]."""
    h = np.asarray(h, f64)
    return np.concatenate([np.asarray(W_Q_i, f64) @ h,
                           rope(np.asarray(W_QR_i, f64) @ h, pos, base)])


def expanded_kv(C: np.ndarray, KR: np.ndarray, W_UK_i: np.ndarray, W_UV_i: np.ndarray):
    """Per-head keys K_i = [W^UK_i c_j || k^R_j] and values V_i = W^UV_i c_j for
    every cached row j: C [L, d_c], KR [L, d_R] -> K [L, d_h + d_R], V [L, d_v]."""
    C = np.asarray(C, f64)
    K = np.concatenate([C @ np.asarray(W_UK_i, f64).T, np.asarray(KR, f64)], axis=1)
    V = C @ np.asarray(W_UV_i, f64).T
    return K, V


def softmax_attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, n_valid: int):
    """a = softmax(scale * K q) over rows j < n_valid; returns (a V, lse, a)."""
    s = scale * (np.asarray(K[:n_valid], f64) @ np.asarray(q, f64))
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    a = e / z
    return a @ np.asarray(V[:n_valid], f64), m + math.log(z), a


# ----------------------------------------------------------------------------
# cache access
# ----------------------------------------------------------------------------
def gather_rows(cache, block_table, page_size: int, b: int, L: int):
    """Logical rows 0..L-1 of sequence b through its block table."""
    j = np.arange(L)
    rows = np.asarray(block_table)[b, j // page_size].astype(np.int64) * page_size + j % page_size
    return np.asarray(np.asarray(cache)[rows], f64)


def pipeline_cache(inp: dict, w) -> np.ndarray:
    """The cache a full-pipeline workload holds: row of position t of sequence
    b is [W^DKV h_t || RoPE(W^KR h_t, t)], stored through the block table."""
    rows = inp["num_pages"] * w.page_size
    cache = np.zeros((rows, w.d_c + w.d_R), dtype=f64)
    for b in range(w.B):
        L = int(inp["seqlens"][b])
        h = np.asarray(inp["h_ctx"][b, :L], f64)
        t = np.arange(L)
        rid = np.asarray(inp["block_table"])[b, t // w.page_size].astype(np.int64) * w.page_size + t % w.page_size
        cache[rid, :w.d_c] = latent(inp["W_DKV"], h)
        cache[rid, w.d_c:] = rope_key(inp["W_KR"], h, t, w.rope_base)
    return cache


def _cache_of(inp, w):
    return inp["cache"] if "cache" in inp else pipeline_cache(inp, w)


# ----------------------------------------------------------------------------
# decode, expanded (the definition)
# ----------------------------------------------------------------------------
def decode_expanded(inp: dict, w, picks=None, cache=None):
    """Non-absorbed decode.

    For every picked (b, r, i): materialise K_i and V_i for the cached rows of
    sequence b, form q_i from h, mask positions j > L_b - s_q + r, softmax,
    and take o = sum_j a_j v_j.  Returns dict (b, r, i) -> (o [d_v], lse).
    ``picks`` None means every (b, r, i).
    """
    cache = _cache_of(inp, w) if cache is None else cache
    if picks is None:
        picks = [(b, r, i) for b in range(w.B) for r in range(w.s_q) for i in range(w.n_h)]
    by_seq = {}
    for (b, r, i) in picks:
        by_seq.setdefault(b, []).append((r, i))
    out = {}
    for b, items in by_seq.items():
        L = int(inp["seqlens"][b])
        rows = gather_rows(cache, inp["block_table"], w.page_size, b, L)
        C, KR = rows[:, :w.d_c], rows[:, w.d_c:]
        heads = sorted({i for _, i in items})
        kv = {i: expanded_kv(C, KR, inp["W_UK"][i], inp["W_UV"][i]) for i in heads}
        for (r, i) in items:
            pos = int(inp["qpos"][b, r])
            q = query_head(inp["W_Q"][i], inp["W_QR"][i], inp["h_q"][b, r], pos, w.rope_base)
            K, V = kv[i]
            o, lse, _ = softmax_attend(q, K, V, w.softmax_scale, n_valid=pos + 1)
            out[(b, r, i)] = (o, lse)
    return out


# ----------------------------------------------------------------------------
# absorbed helper (separate code path, used to check the GPU's u)
# ----------------------------------------------------------------------------
def absorb_weights(W_UK: np.ndarray, W_Q: np.ndarray) -> np.ndarray:
    """W^QK_i = (W^UK_i)^T W^Q_i: [n_h, d_h, d_c] x [n_h, d_h, d_model] -> [n_h, d_c, d_model]."""
    return np.einsum("hkc,hkd->hcd", np.asarray(W_UK, f64), np.asarray(W_Q, f64))


def absorbed_query(inp: dict, w, b: int, r: int, i: int, W_QK_i=None) -> np.ndarray:
    """q^lat_i = W^QK_i h (or W^UK_i^T (W^Q_i h) when W^QK_i is not given),
    concatenated with q^R_i = RoPE(W^QR_i h, pos): [d_c + d_R]."""
    h = np.asarray(inp["h_q"][b, r], f64)
    if W_QK_i is None:
        qlat = np.asarray(inp["W_UK"][i], f64).T @ (np.asarray(inp["W_Q"][i], f64) @ h)
    else:
        qlat = np.asarray(W_QK_i, f64) @ h
    qr = rope(np.asarray(inp["W_QR"][i], f64) @ h, int(inp["qpos"][b, r]), w.rope_base)
    return np.concatenate([qlat, qr])


def decode_absorbed(q: np.ndarray, cache, block_table, seqlens, w, picks=None,
                    with_abs: bool = False, W_UV=None):
    """Absorbed decode from an explicit query tensor q [B, s_q, n_h, d_c + d_R]:
    s_j = q^lat.c_j + q^R.k^R_j, a = softmax(scale s) over j <= L - s_q + r,
    u = sum_j a_j c_j.  Returns dict (b, r, i) -> (u [d_c], lse).

    with_abs: the value is a dict with u, lse and abs_c = sum_j a_j |c_j|
    (the scale against which rounding of the weights a_j is measured); given
    W_UV as well, also o = W^UV_i u and abs_v = sum_j a_j |W^UV_i c_j|."""
    if picks is None:
        picks = [(b, r, i) for b in range(w.B) for r in range(w.s_q) for i in range(w.n_h)]
    by_seq = {}
    for (b, r, i) in picks:
        by_seq.setdefault(b, []).append((r, i))
    out = {}
    for b, items in by_seq.items():
        L = int(seqlens[b])
        rows = gather_rows(cache, block_table, w.page_size, b, L)
        for (r, i) in items:
            n_valid = L - w.s_q + r + 1
            qv = np.asarray(q[b, r, i], f64)
            s = w.softmax_scale * (rows[:n_valid] @ qv)
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            a = e / z
            C = rows[:n_valid, :w.d_c]
            u = a @ C
            lse = m + math.log(z)
            if not with_abs:
                out[(b, r, i)] = (u, lse)
                continue
            d = dict(u=u, lse=lse, abs_c=a @ np.abs(C))
            if W_UV is not None:
                Wi = np.asarray(W_UV[i], f64)
                d["o"] = Wi @ u
                d["abs_v"] = a @ np.abs(C @ Wi.T)
            out[(b, r, i)] = d
    return out


def absorbed_queries(inp: dict, w, b: int, r: int) -> np.ndarray:
    """absorbed_query for every head of row (b, r) at once: q^lat_i =
    W^UK_i^T (W^Q_i h) and q^R_i = RoPE(W^QR_i h, pos), as [n_h, d_c + d_R]."""
    h = np.asarray(inp["h_q"][b, r], f64)
    qn = np.einsum("hkd,d->hk", np.asarray(inp["W_Q"], f64), h)            # W^Q_i h
    qlat = np.einsum("hkc,hk->hc", np.asarray(inp["W_UK"], f64), qn)      # W^UK_i^T (.)
    pos = int(inp["qpos"][b, r])
    qr = np.einsum("hkd,d->hk", np.asarray(inp["W_QR"], f64), h)
    qr = np.stack([rope(x, pos, w.rope_base) for x in qr])
    return np.concatenate([qlat, qr], axis=1)


def decode_absorbed_seq(q_b: np.ndarray, cache, block_table, L: int, b: int, w,
                        want_abs: bool = False):
    """decode_absorbed for every query row and head of sequence b at once, as
    plain fp64 matrix products over all heads: q_b [s_q, n_h, d_c + d_R],
    S = rows . q^T, row r masked past position L - s_q + r, a = softmax(scale S)
    per (r, head), u = a^T C.  Returns (u [s_q, n_h, d_c], lse [s_q, n_h]) and,
    with want_abs, abs_c = a^T |C| [s_q, n_h, d_c] as a third value."""
    rows = gather_rows(cache, block_table, w.page_size, b, L)
    C = rows[:, :w.d_c]
    absC = np.abs(C) if want_abs else None
    s_q = q_b.shape[0]
    u = np.empty((s_q, q_b.shape[1], w.d_c))
    lse = np.empty((s_q, q_b.shape[1]))
    abs_c = np.empty_like(u) if want_abs else None
    for r in range(s_q):
        n_valid = L - s_q + r + 1
        S = w.softmax_scale * (rows[:n_valid] @ np.asarray(q_b[r], f64).T)   # [n_valid, n_h]
        m = S.max(axis=0)
        e = np.exp(S - m)
        z = e.sum(axis=0)
        a = e / z
        u[r] = a.T @ C[:n_valid]
        lse[r] = m + np.log(z)
        if want_abs:
            abs_c[r] = a.T @ absC[:n_valid]
    return (u, lse, abs_c) if want_abs else (u, lse)


def absorbed_queries_all(inp: dict, w) -> np.ndarray:
    """absorbed_queries for every (b, r): [B, s_q, n_h, d_c + d_R].  The same
    two products per head, W^UK_i^T (W^Q_i h) and RoPE(W^QR_i h, pos), taken
    over all query rows at once."""
    H = np.asarray(inp["h_q"], f64).reshape(w.B * w.s_q, w.d_model)             # [T, d_model]
    qn = np.tensordot(H, np.asarray(inp["W_Q"], f64), axes=([1], [2]))          # [T, n_h, d_h]
    qlat = np.einsum("thk,hkc->thc", qn, np.asarray(inp["W_UK"], f64))          # [T, n_h, d_c]
    qr = np.tensordot(H, np.asarray(inp["W_QR"], f64), axes=([1], [2]))         # [T, n_h, d_R]
    pos = np.asarray(inp["qpos"]).reshape(-1)
    for t in range(qr.shape[0]):
        qr[t] = np.stack([rope(x, int(pos[t]), w.rope_base) for x in qr[t]])
    return np.concatenate([qlat, qr], axis=2).reshape(w.B, w.s_q, w.n_h, w.d_c + w.d_R)


def output_projection(o: np.ndarray, W_O: np.ndarray) -> np.ndarray:
    """y_t = W^O concat_i(o_{t,i}): the heads' outputs concatenated and
    projected to the hidden size ("Attention-head anatomy" section 5, the
    output side W^O that W^UV folds into).  o [T, n_h, d_v],
    W^O [d_model, n_h * d_v] -> y [T, d_model]."""
    o = np.asarray(o, f64)
    return o.reshape(o.shape[0], -1) @ np.asarray(W_O, f64).T


def up_project(u: np.ndarray, W_UV: np.ndarray) -> np.ndarray:
    """o_i = W^UV_i u_i: u [..., n_h, d_c], W^UV [n_h, d_v, d_c] -> [..., n_h, d_v]."""
    return np.einsum("...hc,hvc->...hv", np.asarray(u, f64), np.asarray(W_UV, f64))


# ----------------------------------------------------------------------------
# GQLA's GQA path (GQLA summary, abstract and method paragraphs): heads of a
# group share W^UK_g and W^UV_g, so the cache can hold per group the expanded
# key K^C_g = W^UK_g c and value V_g = W^UV_g c; the RoPE key stays shared.
# ----------------------------------------------------------------------------
def expand_gqa_cache(cache, W_UK_g, W_UV_g, d_c: int) -> tuple:
    """Per-group expanded cache from a latent cache [rows, d_c + d_R]:
    kv [rows, n_g, d_h + d_v] = [c W^UK_g^T || c W^UV_g^T] and the shared
    RoPE keys [rows, d_R]."""
    cache = np.asarray(cache, f64)
    C, KR = cache[:, :d_c], cache[:, d_c:]
    K = np.einsum("rc,gkc->rgk", C, np.asarray(W_UK_g, f64))
    V = np.einsum("rc,gvc->rgv", C, np.asarray(W_UV_g, f64))
    return np.concatenate([K, V], axis=2), KR


def decode_gqa(q, kv, k_rope, block_table, seqlens, w, n_g: int, picks=None):
    """GQA decode over the per-group expanded cache: head i uses group
    g = i // (n_h / n_g); s_j = q^nope . K^C_g[j] + q^R . k^R[j] for
    j <= L - s_q + r, a = softmax(scale s), o = sum_j a_j V_g[j].
    Returns dict (b, r, i) -> (o [d_v], lse)."""
    hpg = w.n_h // n_g
    if picks is None:
        picks = [(b, r, i) for b in range(w.B) for r in range(w.s_q) for i in range(w.n_h)]
    out = {}
    kv = np.asarray(kv)
    k_rope = np.asarray(k_rope)
    for (b, r, i) in picks:
        L = int(seqlens[b])
        j = np.arange(L)
        rows = np.asarray(block_table)[b, j // w.page_size].astype(np.int64) * w.page_size + j % w.page_size
        g = i // hpg
        K = np.asarray(kv[rows, g, :w.d_h], f64)
        V = np.asarray(kv[rows, g, w.d_h:], f64)
        KR = np.asarray(k_rope[rows], f64)
        qv = np.asarray(q[b, r, i], f64)
        n_valid = L - w.s_q + r + 1
        s = w.softmax_scale * (K[:n_valid] @ qv[:w.d_h] + KR[:n_valid] @ qv[w.d_h:])
        m = s.max()
        e = np.exp(s - m)
        z = e.sum()
        out[(b, r, i)] = ((e / z) @ V[:n_valid], m + math.log(z))
    return out
