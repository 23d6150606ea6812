"""The five workloads at full size, in the launch configuration the bench
times (automatic KV chunking, fp32 u).  u and lse are compared with the
oracle's absorbed helper for every (sequence, query row, head); o = W^UV u
is compared with the non-absorbed oracle on a seeded sample of
(sequence, head) picks, which it computes one by one."""
import numpy as np
import pytest
import torch

from gpu_pipeline import (ATOL_REL, assert_parity, assert_tight, check_absorbed, check_expanded,
                          f64, lse_err, run_pipeline, tight_u_bound, to_dev)
from mla_latent_kv_23_b200 import mla, synth
from oracle import mla_oracle as orc

pytestmark = pytest.mark.gpu


def sample_picks(w, inp, n_seq, n_head, seed):
    rng = np.random.default_rng(seed)
    bs = sorted(rng.choice(w.B, size=min(n_seq, w.B), replace=False).tolist())
    # always include the longest and the shortest sequence
    bs = sorted(set(bs) | {int(np.argmax(inp["seqlens"])), int(np.argmin(inp["seqlens"]))})
    picks = []
    for b in bs:
        for i in sorted(set(rng.choice(w.n_h, size=n_head, replace=False).tolist()) | {0, w.n_h - 1}):
            for r in range(w.s_q):
                picks.append((b, r, i))
    return picks


def check_every_row(w, inp, out, q_of):
    """u and lse of every (b, r, i) against the absorbed helper on the query
    q_of(b) [s_q, n_h, d_c + d_R]: the elementwise tolerance and, when the
    query is the one the GPU used, the bound derived from the kernel's
    rounding.  Returns (worst u error, worst lse error in allowance units,
    worst u error over its tight bound, rows checked)."""
    u, lse = f64(out["u"]), f64(out["lse"])
    worst_u = worst_l = worst_t = 0.0
    n = 0
    for b in range(w.B):
        ur, lr, ac = orc.decode_absorbed_seq(q_of(b), inp["cache"], inp["block_table"],
                                             int(inp["seqlens"][b]), b, w, want_abs=True)
        worst_u = max(worst_u, float(np.max(np.abs(u[b] - ur) / (1 + np.abs(ur)))))
        worst_t = max(worst_t, float(np.max(np.abs(u[b] - ur) / tight_u_bound(ur, ac))))
        worst_l = max(worst_l, max(lse_err(g, e) for g, e in zip(lse[b].ravel(), lr.ravel())))
        n += w.s_q * w.n_h
    return worst_u, worst_l, worst_t, n


@pytest.mark.parametrize("name", ["v3", "ragged", "mtp"])
def test_full_size_config(name):
    w = synth.config(name)
    inp = synth.draw(w)
    out = run_pipeline(w, inp)
    assert out["u"].dtype == torch.float32
    for t in (out["u"], out["lse"], out["o"]):
        assert torch.isfinite(t.float()).all()
    # every row: the oracle's own fp64 query (W^UK^T (W^Q h), RoPE'd W^QR h)
    wu, wl, _, n = check_every_row(
        w, inp, out, lambda b: np.stack([orc.absorbed_queries(inp, w, b, r) for r in range(w.s_q)]))
    print(f"{name}: every row: u {wu:.3e} lse {wl:.3f} (allowance units), n = {n}")
    assert n == w.B * w.s_q * w.n_h
    assert wu <= ATOL_REL and wl <= 1.0
    # o through the non-absorbed definition on a sample
    picks = sample_picks(w, inp, 3, 3, seed=w.seed)
    assert_parity(check_expanded(w, inp, out, picks))


def test_long_context_stress():
    """131072 tokens per sequence, 1% of cached rows scaled x8, >= 64 KV
    chunks.  The x8 rows put the top logits near 25, where rounding q itself
    to bf16 moves u by up to ~0.06 (1 + |u|), so the decode is checked on its
    own bf16 inputs: q comes from the generator and the oracle runs on the
    same q.  Every row's u and lse meet the elementwise tolerance and the
    bound derived from the kernel's rounding; o = W^UV u meets the
    elementwise tolerance and its derived bound on a sample."""
    w = synth.config("long")
    inp = synth.draw(w)
    q = synth.random_q(w)
    out = run_pipeline(w, inp, q=to_dev(q, w))
    p = mla.decode_params(out["q"], out["cache"], out["bt"], out["seqlens"], out["u"], out["lse"],
                          w.page_size, w.d_R, w.softmax_scale)
    _, chunks = mla.mla_decode_kernel_info(p)
    assert chunks >= 64
    wu, wl, wt, n = check_every_row(w, inp, out, lambda b: q[b])
    print(f"long: every row: u {wu:.3e} lse {wl:.3f} tight {wt:.3f}, n = {n}")
    assert n == w.B * w.s_q * w.n_h
    assert wu <= ATOL_REL and wl <= 1.0 and wt <= 1.0
    picks = sample_picks(w, inp, 4, 6, seed=w.seed)
    res = check_absorbed(w, q, inp, out, picks, W_UV=inp["W_UV"])
    print("long-context stress, sampled o:", res)
    assert_tight(res)


def test_tiny_config_all_outputs():
    # fp32 throughout: the decode runs on the small-latent tensor-core kernel
    # (tf32) and the up-projection as tf32 MMAs
    w = synth.config("tiny")
    inp = synth.draw(w)
    out = run_pipeline(w, inp)
    p = mla.decode_params(out["q"], out["cache"], out["bt"], out["seqlens"], out["u"], out["lse"],
                          w.page_size, w.d_R, w.softmax_scale)
    tc, _ = mla.mla_decode_kernel_info(p)
    assert tc == 1
    res = check_expanded(w, inp, out)
    assert res["n"] == w.B * w.s_q * w.n_h
    assert_parity(res)
