"""Runs the CUDA path through the C ABI on inputs from the seeded generator,
and compares results with the oracle.  Used by the -m gpu tests only."""
from __future__ import annotations

import numpy as np
import torch

from mla_latent_kv_23_b200 import mla, synth
from oracle import mla_oracle as orc

from mla_latent_kv_23_b200.device_inputs import (absorb_and_query, build_cache, tdtype,  # noqa: F401
                                                 to_dev, to_dev_i32)

# target tolerances: elementwise |gpu - oracle| <= ATOL_REL * (1 + |oracle|);
# softmax statistics within LSE_REL relative.  "Relative" is taken against
# max(|lse|, 1): lse is the log of a sum, and a row whose lse is near 0 (one
# cached token with a score near 0) would otherwise be asked for more digits
# than its scores carry (tf32 scores, from fp32 tensors, hold about 1e-4 of
# absolute error).
ATOL_REL = 2e-2
LSE_REL = 1e-3


def lse_err(got, ref):
    """Error of an lse in units of its allowance (<= 1 passes)."""
    return abs(got - ref) / (LSE_REL * max(abs(ref), 1.0))


def run_pipeline(w, inp, num_splits=0, q=None, device="cuda", u_dtype=None):
    """absorb -> query -> (append) -> decode -> up-projection, all through
    libmla; u is fp32 unless u_dtype says otherwise."""
    if q is None:
        q, _ = absorb_and_query(w, inp, device)
    cache, bt = build_cache(w, inp, device)
    seqlens = to_dev_i32(inp["seqlens"], device)
    u, lse = mla.decode(q, cache, bt, seqlens, w.page_size, w.d_R, w.softmax_scale,
                        num_splits=num_splits, u_dtype=u_dtype)
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


# Tighter bounds for decode-only comparisons on identical inputs, derived from
# the kernel's arithmetic.  bf16 has 8 significant bits: rounding to it moves
# a value by at most 2^-8 of itself.  Scores, exponentials, sums and every
# accumulation are fp32; the softmax weights P_j are rounded to bf16 before
# the P.C contraction and u is normalised by the sum of those rounded weights.
# With a_j the exact weights and d_j the relative rounding of P_j,
#   u' - u = sum_j a_j d_j (c_j - u) / (1 + sum_j a_j d_j),
# so |du_k| <= 2^-8 (abs_c_k + |u_k|) (1 + 2^-7), abs_c = sum_j a_j |c_j|.
# A bf16 u adds 2^-8 |u_k| for its own rounding and 2^-8 abs_c_k for the bf16
# partials of split rows (each partial within 2^-8 of itself; the split
# weights sum to 1).  Through o = W^UV u the weight term becomes
# 2^-8 (abs_v + |o|), abs_v = sum_j a_j |W^UV c_j|, and o's bf16 rounding
# adds 2^-8 |o|; with an fp32 u the up-projection splits u into two bf16
# terms (error 2^-16 |u|), with a bf16 u it adds 2^-8 |W^UV| (abs_c + |u|).
# With an fp32 u the partials of split rows are fp16 (11 significant bits):
# they add 2^-11 abs_c_k to u and 2^-11 |W^UV| abs_c to o.
# The checks allow 1.5x these (fp32 accumulation order, the (1 + 2^-7)).
TIGHT_SLACK = 1.5


def tight_u_bound(u_ref, abs_c, u_fp32=True):
    b = 2.0 ** -8 * (abs_c + np.abs(u_ref))
    if u_fp32:
        b = b + 2.0 ** -11 * abs_c
    else:
        b = b + 2.0 ** -8 * (abs_c + np.abs(u_ref))
    return TIGHT_SLACK * b + 1e-6


def tight_o_bound(o_ref, abs_v, W_i, u_ref, abs_c=None, u_fp32=True):
    b = 2.0 ** -8 * (abs_v + 2.0 * np.abs(o_ref))
    if u_fp32:
        b = b + 2.0 ** -11 * (np.abs(W_i) @ abs_c)
    else:
        b = b + 2.0 ** -8 * (np.abs(W_i) @ (abs_c + np.abs(u_ref)))
    return TIGHT_SLACK * b + 1e-6


def check_absorbed(w, q, inp, out, picks, W_UV=None):
    """u / lse / o of a decode run on the generator's q against the oracle's
    absorbed helper (itself pinned to the expanded definition)."""
    ref = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w, picks,
                              with_abs=True, W_UV=W_UV)
    import torch
    u_fp32 = out["u"].dtype == torch.float32
    u, lse = f64(out["u"]), f64(out["lse"])
    o = f64(out["o"]) if out.get("o") is not None else None
    res = dict(o=0.0, u=0.0, lse=0.0, tight=0.0, tight_o=0.0, n=len(ref))
    for (b, r, i), d in ref.items():
        u_ref, lse_ref = d["u"], d["lse"]
        res["u"] = max(res["u"], float(np.max(np.abs(u[b, r, i] - u_ref) / (1 + np.abs(u_ref)))))
        res["tight"] = max(res["tight"], float(np.max(np.abs(u[b, r, i] - u_ref) /
                                                      tight_u_bound(u_ref, d["abs_c"], u_fp32))))
        res["lse"] = max(res["lse"], lse_err(lse[b, r, i], lse_ref))
        if o is not None and W_UV is not None:
            o_ref = d["o"]
            err = np.abs(o[b, r, i] - o_ref)
            res["o"] = max(res["o"], float(np.max(err / (1 + np.abs(o_ref)))))
            bound = tight_o_bound(o_ref, d["abs_v"], np.asarray(W_UV[i], np.float64), u_ref,
                                  d["abs_c"], u_fp32)
            res["tight_o"] = max(res["tight_o"], float(np.max(err / bound)))
    return res


def assert_tight(res):
    """The elementwise tolerance on o, u and lse, and the bounds derived from
    the kernel's rounding on u and o."""
    assert_parity(res)
    assert res["tight"] <= 1.0, res
    assert res["tight_o"] <= 1.0, res


def assert_parity(res):
    assert res["o"] <= ATOL_REL, res
    assert res["u"] <= ATOL_REL, res
    assert res["lse"] <= 1.0, res
