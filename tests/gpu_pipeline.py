"""Runs the CUDA path through the C ABI on inputs from the seeded generator,
and compares results with the oracle.  Used by the -m gpu tests only."""
from __future__ import annotations

import numpy as np
import torch

from mla_latent_kv_23_b200 import mla, synth
from oracle import mla_oracle as orc

# target tolerances: elementwise |gpu - oracle| <= ATOL_REL * (1 + |oracle|);
# softmax statistics within LSE_REL relative.  "Relative" is taken against
# max(|lse|, 1): a row with a single cached token has lse = its own score,
# which can be ~0, where a purely relative test has no meaning.
ATOL_REL = 2e-2
LSE_REL = 1e-3


def lse_err(got, ref):
    return abs(got - ref) / max(abs(ref), 1.0)


def tdtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_dev(x, w, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device).to(tdtype(w))


def to_dev_i32(x, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def absorb_and_query(w, inp, device="cuda"):
    """W_QK = absorb(W_UK, W_Q); q = [W_QK h || RoPE(W_QR h, pos)] on the GPU."""
    W_UK, W_Q, W_QR = (to_dev(inp[k], w, device) for k in ("W_UK", "W_Q", "W_QR"))
    W_QK = torch.empty((w.n_h, w.d_c, w.d_model), dtype=tdtype(w), device=device)
    mla.mla_absorb_weights(W_UK, W_Q, W_QK)
    del W_Q
    h = to_dev(inp["h_q"].reshape(w.B * w.s_q, w.d_model), w, device)
    pos = to_dev_i32(inp["qpos"].reshape(-1), device)
    q = torch.empty((w.B * w.s_q, w.n_h, w.width), dtype=tdtype(w), device=device)
    mla.mla_form_query(h, W_QK, W_QR, pos, q, rope_base=w.rope_base)
    return q.view(w.B, w.s_q, w.n_h, w.width), W_QK


def build_cache(w, inp, device="cuda"):
    """The paged cache on the GPU: copied from the generator, or (full
    pipeline) appended token by token with mla_append_latent."""
    rows = inp["num_pages"] * w.page_size
    bt = to_dev_i32(inp["block_table"], device)
    if "cache" in inp:
        return to_dev(inp["cache"], w, device), bt
    cache = torch.zeros((rows, w.width), dtype=tdtype(w), device=device)
    seq = np.concatenate([np.full(int(L), b, np.int32) for b, L in enumerate(inp["seqlens"])])
    pos = np.concatenate([np.arange(int(L), dtype=np.int32) for L in inp["seqlens"]])
    h = np.concatenate([inp["h_ctx"][b, :int(L)] for b, L in enumerate(inp["seqlens"])])
    mla.mla_append_latent(to_dev(h, w, device), to_dev(inp["W_DKV"], w, device),
                          to_dev(inp["W_KR"], w, device), to_dev_i32(seq, device),
                          to_dev_i32(pos, device), bt, cache, w.page_size, rope_base=w.rope_base)
    return cache, bt


def run_pipeline(w, inp, num_splits=0, q=None, device="cuda"):
    """absorb -> query -> (append) -> decode -> up-projection, all through libmla."""
    if q is None:
        q, _ = absorb_and_query(w, inp, device)
    cache, bt = build_cache(w, inp, device)
    seqlens = to_dev_i32(inp["seqlens"], device)
    u, lse = mla.decode(q, cache, bt, seqlens, w.page_size, w.d_R, w.softmax_scale,
                        num_splits=num_splits)
    W_UV = to_dev(inp["W_UV"], w, device) if "W_UV" in inp else None
    o = None
    if W_UV is not None:
        o = torch.empty((w.B * w.s_q, w.n_h, w.d_v), dtype=tdtype(w), device=device)
        mla.mla_up_proj(u.view(w.B * w.s_q, w.n_h, w.d_c), W_UV, o)
        o = o.view(w.B, w.s_q, w.n_h, w.d_v)
    mla.mla_check_device_errors()
    return dict(q=q, u=u, lse=lse, o=o, cache=cache, bt=bt, seqlens=seqlens)


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_expanded(w, inp, out, picks=None):
    """o and lse against the non-absorbed oracle; u against the oracle's
    absorbed helper (its own fp64 query, never the GPU's)."""
    ref = orc.decode_expanded(inp, w, picks)
    o, lse, u = f64(out["o"]), f64(out["lse"]), f64(out["u"])
    qs = {}
    worst_o = worst_lse = worst_u = 0.0
    abs_picks = list(ref.keys())
    qa = np.zeros((w.B, w.s_q, w.n_h, w.width))
    for (b, r, i) in abs_picks:
        qa[b, r, i] = orc.absorbed_query(inp, w, b, r, i)
    cache = inp["cache"] if "cache" in inp else orc.pipeline_cache(inp, w)
    uref = orc.decode_absorbed(qa, cache, inp["block_table"], inp["seqlens"], w, abs_picks)
    for key, (o_ref, lse_ref) in ref.items():
        b, r, i = key
        eo = np.abs(o[b, r, i] - o_ref) / (1 + np.abs(o_ref))
        worst_o = max(worst_o, float(eo.max()))
        worst_lse = max(worst_lse, lse_err(lse[b, r, i], lse_ref))
        u_ref, lse_a = uref[key]
        eu = np.abs(u[b, r, i] - u_ref) / (1 + np.abs(u_ref))
        worst_u = max(worst_u, float(eu.max()))
        qs[key] = True
    return dict(o=worst_o, lse=worst_lse, u=worst_u, n=len(ref))


# Tighter bounds for decode-only comparisons on identical bf16 inputs, derived
# from the kernel's arithmetic: each softmax weight is rounded to bf16 before
# the P.C contraction (relative error <= 2^-9, normalised by the sum of the
# rounded weights), u is stored in bf16 (relative error <= 2^-9), and the
# up-projection reads that bf16 u and stores o in bf16; scores, exponentials
# and every accumulation are fp32.  So, up to fp32 terms,
#   |du_k| <= 2^-8 sum_j a_j |c_jk| + 2^-9 |u_k|
#   |do_k| <= 2^-8 sum_j a_j |(W c_j)_k| + 2^-9 sum_c |W_kc| |u_c| + 2^-9 |o_k|
# (a weight error moves a whole cached row, so it reaches o through W^UV).
# The checks allow 2x these.
def tight_u_bound(u_ref, abs_c):
    """Rounding budget of the bf16 path for u_i = sum_j a_j c_j, with
    abs_c = sum_j a_j |c_j|: the bf16 weights P (relative 2^-9 each, so at most
    2^-9 abs_c), the bf16 split partials the combine stage merges (each within
    2^-9 of itself, and the split weights sum to 1, so at most 2^-9 abs_c
    again) and the final bf16 u (2^-9 |u|); doubled for fp32 accumulation
    order."""
    return 2.0 * (2.0 ** -8 * abs_c + 2.0 ** -9 * np.abs(u_ref)) + 1e-6


def tight_o_bound(o_ref, abs_v, W_i, u_ref):
    return 2.0 * (2.0 ** -8 * abs_v + 2.0 ** -9 * (np.abs(W_i) @ np.abs(u_ref)) +
                  2.0 ** -9 * np.abs(o_ref)) + 1e-6


def check_absorbed(w, q, inp, out, picks, W_UV=None):
    """u / lse / o of a decode run on the generator's q against the oracle's
    absorbed helper (itself pinned to the expanded definition)."""
    ref = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w, picks,
                              with_abs=True, W_UV=W_UV)
    u, lse = f64(out["u"]), f64(out["lse"])
    o = f64(out["o"]) if out.get("o") is not None else None
    res = dict(o=0.0, u=0.0, lse=0.0, tight=0.0, tight_o=0.0, n=len(ref))
    for (b, r, i), d in ref.items():
        u_ref, lse_ref = d["u"], d["lse"]
        res["u"] = max(res["u"], float(np.max(np.abs(u[b, r, i] - u_ref) / (1 + np.abs(u_ref)))))
        res["tight"] = max(res["tight"], float(np.max(np.abs(u[b, r, i] - u_ref) /
                                                      tight_u_bound(u_ref, d["abs_c"]))))
        res["lse"] = max(res["lse"], lse_err(lse[b, r, i], lse_ref))
        if o is not None and W_UV is not None:
            o_ref = d["o"]
            err = np.abs(o[b, r, i] - o_ref)
            res["o"] = max(res["o"], float(np.max(err / (1 + np.abs(o_ref)))))
            bound = tight_o_bound(o_ref, d["abs_v"], np.asarray(W_UV[i], np.float64), u_ref)
            res["tight_o"] = max(res["tight_o"], float(np.max(err / bound)))
    return res


def assert_tight(res, o_elementwise=True):
    """Tight bounds on u (and o when present); the elementwise tolerance on
    u and lse always, and on o unless o_elementwise is False."""
    assert res["u"] <= ATOL_REL, res
    assert res["lse"] <= LSE_REL, res
    if o_elementwise:
        assert res["o"] <= ATOL_REL, res
    assert res["tight"] <= 1.0, res
    assert res["tight_o"] <= 1.0, res


def assert_parity(res):
    assert res["o"] <= ATOL_REL, res
    assert res["u"] <= ATOL_REL, res
    assert res["lse"] <= LSE_REL, res
