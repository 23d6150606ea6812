"""Device-side preparation of a seeded workload's inputs through libmla.

Moves the generator's arrays (mla_latent_kv_23_b200.synth) to the GPU and
runs the setup calls of the C ABI on them: weight absorption and query
formation (mla_absorb_weights, mla_form_query), and for the full-pipeline
workload the latent append into the paged cache (mla_append_latent).  Used
by bench.py and by the GPU tests; it only moves data and calls the library,
so it holds none of the attention arithmetic.
"""
from __future__ import annotations

import numpy as np

from . import mla


def tdtype(w):
    import torch
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_dev(x, w, device="cuda"):
    """A float array of the generator (exact in the workload's storage type)
    as a device tensor of that type."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device).to(tdtype(w))


def to_dev_i32(x, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def absorb_and_query(w, inp, device="cuda"):
    """W_QK = absorb(W_UK, W_Q); q = [W_QK h || RoPE(W_QR h, pos)], both
    computed by the library.  Returns (q [B, s_q, n_h, d_c + d_R], W_QK)."""
    import torch
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
    pipeline) appended token by token with mla_append_latent.  Returns
    (cache, block_table)."""
    import torch
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
