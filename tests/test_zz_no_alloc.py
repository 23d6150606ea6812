"""mla_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers (a host framework that owns all device memory, a plugin
interface that passes no workspace) cannot give the library scratch space.
For them mla_decode_noalloc uses a fixed array inside the library instead
of a workspace.  This file checks, through the C ABI, that it returns what
mla_decode returns bit for bit (both run the same kernels on the same
chunking, so any difference would be stale data in the shared array), on
two calls in a row with different inputs (the second call finds the first
call's data still in the shared array), and that parameters needing more
than the array's 32 MiB are refused up front.
The file is named to run last.
"""
import numpy as np
import pytest
import torch

from gpu_pipeline import to_dev, to_dev_i32
from mla_latent_kv_23_b200 import mla, synth

pytestmark = pytest.mark.gpu

NOALLOC_LIMIT = 32 << 20


def _inputs(seqlens, s_q, seed):
    w = synth.Workload(name="noalloc", B=len(seqlens), s_q=s_q, n_h=128, d_model=64, d_c=512,
                       d_h=128, d_v=128, d_R=64, page_size=64, dtype="bf16", seqlens=seqlens,
                       block_table="permuted", scale=1 / np.sqrt(192.0), seed=seed)
    inp = synth.draw(w, with_weights=False)
    return (w, to_dev(synth.random_q(w), w), to_dev(inp["cache"], w),
            to_dev_i32(inp["block_table"]), to_dev_i32(inp["seqlens"]))


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    cases = [((700, 64, 1999), 1, 31), ((300, 5000, 2, 129), 2, 32)]
    for seqlens, s_q, seed in cases:
        w, q, cache, bt, sl = _inputs(seqlens, s_q, seed)
        u_ref, lse_ref = mla.decode(q, cache, bt, sl, w.page_size, w.d_R, w.softmax_scale)
        u = torch.full_like(u_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        p = mla.decode_params(q, cache, bt, sl, u, lse, w.page_size, w.d_R, w.softmax_scale)
        assert mla.mla_decode_workspace_size(p) <= NOALLOC_LIMIT
        mla.mla_decode_noalloc(p)
        torch.cuda.synchronize()
        assert mla.mla_check_device_errors() == 0
        assert torch.equal(u, u_ref) and torch.equal(lse, lse_ref)


def test_noalloc_refuses_parameters_beyond_its_array():
    B = 300   # (B + chunks) partial rows of 128 x 512 fp32 need well over 32 MiB
    q = torch.zeros((B, 1, 128, 576), dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((64, 576), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
    sl = torch.ones((B,), dtype=torch.int32, device="cuda")
    u = torch.empty((B, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    p = mla.decode_params(q, cache, bt, sl, u, None, 64, 64, 0.07)
    assert mla.mla_decode_workspace_size(p) > NOALLOC_LIMIT
    with pytest.raises(mla.MLAError) as e:
        mla.mla_decode_noalloc(p)
    assert e.value.status == 4   # MLA_ERR_WORKSPACE_TOO_SMALL
