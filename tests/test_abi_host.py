"""Host-only checks of the C ABI: the library loads, exports every function
include/mla.h declares, and rejects bad arguments before touching a device.
No kernel is launched here."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_23_b200 import mla

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mla.h")
INVALID, UNSUPPORTED, OK = 1, 2, 0


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(mla_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(mla.LIB_PATH):
        from mla_latent_kv_23_b200 import build
        build.build()
    return mla.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mla.SIGNATURES), set(names) ^ set(mla.SIGNATURES)


def test_status_strings(lib):
    for s in range(6):
        assert mla.mla_status_string(s)


def params(**kw):
    base = dict(q=16, kv_cache=32, block_table=48, seqlens=64, u=80, lse=96, B=2, s_q=1, n_h=128,
                d_c=512, d_R=64, page_size=64, max_pages_per_seq=4, num_pages=8,
                softmax_scale=0.07, dtype=mla.MLA_DTYPE_BF16, num_splits=0)
    base.update(kw)
    return mla.DecodeParams(**base)


@pytest.mark.parametrize("kw,want", [
    (dict(s_q=0), INVALID), (dict(s_q=3), UNSUPPORTED), (dict(n_h=0), INVALID),
    (dict(n_h=129), UNSUPPORTED), (dict(d_c=12), INVALID), (dict(d_c=1024), UNSUPPORTED),
    (dict(d_R=7), INVALID), (dict(d_R=128), UNSUPPORTED), (dict(page_size=63), INVALID),
    (dict(page_size=0), INVALID), (dict(max_pages_per_seq=0), INVALID), (dict(num_pages=0), INVALID),
    (dict(softmax_scale=float("nan")), INVALID), (dict(softmax_scale=float("inf")), INVALID),
    (dict(softmax_scale=0.0), INVALID), (dict(softmax_scale=-0.1), INVALID),
    (dict(dtype=7), INVALID), (dict(num_splits=-1), INVALID), (dict(B=-1), INVALID),
    (dict(q=None), INVALID), (dict(kv_cache=None), INVALID), (dict(u=None), INVALID),
    (dict(block_table=None), INVALID), (dict(seqlens=None), INVALID),
    (dict(q=17), INVALID), (dict(kv_cache=40), INVALID), (dict(lse=4), INVALID),
])
def test_decode_rejects_bad_arguments(lib, kw, want):
    p = params(**kw)
    for fn in ("mla_decode", "mla_decode_plan", "mla_decode_attend", "mla_decode_combine"):
        assert getattr(lib, fn)(ctypes.byref(p), None, 0, None) == want, fn


def test_decode_null_params(lib):
    assert lib.mla_decode(None, None, 0, None) == INVALID
    n = ctypes.c_size_t(0)
    assert lib.mla_decode_workspace_size(None, ctypes.byref(n)) == INVALID
    assert lib.mla_decode_workspace_size(ctypes.byref(params()), None) == INVALID


def test_empty_batch_is_a_noop(lib):
    p = params(B=0, q=None, kv_cache=None, u=None, block_table=None, seqlens=None)
    assert lib.mla_decode(ctypes.byref(p), None, 0, None) == OK


def test_other_entry_points_reject_bad_arguments(lib):
    assert lib.mla_absorb_weights(None, 16, 32, 128, 128, 512, 7168, 0, None) == INVALID
    assert lib.mla_absorb_weights(16, 32, 48, 0, 128, 512, 7168, 0, None) == INVALID
    assert lib.mla_absorb_weights(16, 32, 48, 128, 128, 512, 7168, 9, None) == INVALID
    assert lib.mla_up_proj(16, 32, 48, 4, 0, 512, 128, 0, 0, None) == INVALID
    assert lib.mla_up_proj(None, 32, 48, 4, 128, 512, 128, 0, 0, None) == INVALID
    assert lib.mla_up_proj(16, 32, 48, 0, 128, 512, 128, 0, 0, None) == OK      # T = 0: nothing to do
    assert lib.mla_up_proj(16, 32, 48, 4, 128, 512, 128, 0, 1, None) == INVALID  # bf16 u, fp32 W
    assert lib.mla_up_proj(16, 32, 48, 4, 128, 512, 128, 3, 0, None) == INVALID  # u dtype
    assert lib.mla_up_proj(16, 32, 48, 4, 128, 512, 129, 1, 0, None) == UNSUPPORTED  # d_v > 128
    assert lib.mla_up_proj(16, 32, 48, 4, 128, 96, 128, 1, 0, None) == UNSUPPORTED   # bf16 d_c % 64
    assert lib.mla_form_query(16, 32, 48, 64, 80, 4, 128, 7168, 512, 63, 1e4, 0, None, 0,
                              None) == INVALID
    assert lib.mla_form_query(16, 32, 48, 64, 80, 4, 128, 7168, 512, 64, -1.0, 0, None, 0,
                              None) == INVALID
    assert lib.mla_form_query(16, 32, 48, 64, 80, 0, 128, 7168, 512, 64, 1e4, 0, None, 0,
                              None) == OK
    assert lib.mla_append_latent(16, 32, 48, 64, 80, 96, 4, 0, 8, 112, 4, 256, 64, 16, 1e4, 0,
                                 None, 0, None) == INVALID
    assert lib.mla_append_latent(16, 32, 48, 64, 80, 96, 4, 64, 8, None, 4, 256, 64, 16, 1e4, 0,
                                 None, 0, None) == INVALID
    # fused query formation: odd d_R, null weights, and shapes outside the kernel
    assert lib.mla_form_query_fused(16, 32, 48, 64, 80, 96, 4, 128, 128, 7168, 512, 63, 1e4,
                                    None, 0, None) == INVALID
    assert lib.mla_form_query_fused(16, None, 48, 64, 80, 96, 4, 128, 128, 7168, 512, 64, 1e4,
                                    None, 0, None) == INVALID
    assert lib.mla_form_query_fused(16, 32, 48, 64, 80, 96, 4, 128, 64, 7168, 512, 64, 1e4,
                                    None, 0, None) == UNSUPPORTED          # d_h != 128
    assert lib.mla_form_query_fused(16, 32, 48, 64, 80, 96, 0, 128, 128, 7168, 512, 64, 1e4,
                                    None, 0, None) == OK                   # T = 0
    # output projection: K not a multiple of 64; fold: null weights
    assert lib.mla_output_projection(16, 0, 32, 48, 4, 100, 7168, None, 0, None) == UNSUPPORTED
    assert lib.mla_output_projection(16, 5, 32, 48, 4, 128, 7168, None, 0, None) == INVALID
    assert lib.mla_fold_output_weights(None, 32, 48, 128, 128, 512, 7168, 0, None) == INVALID
    n = ctypes.c_size_t(0)
    assert lib.mla_projection_workspace_size(16384, 8192, 16, 0, ctypes.byref(n)) == OK
    assert n.value >= (128 + 64) * 128 * 64 * 4
    assert lib.mla_projection_workspace_size(-1, 0, 16, 0, ctypes.byref(n)) == INVALID


def test_binding_refuses_host_tensors():
    # the kernels read device memory only: host tensors never reach the library
    import torch
    t = torch.zeros(16)
    with pytest.raises(ValueError):
        mla._ptr(t)
    assert mla._ptr(None) is None


def test_merge_binding_refuses_non_fp32_statistics():
    # the merge kernel reads lse words as fp32; other dtypes are refused before
    # any pointer is taken
    import torch
    u_parts = torch.zeros((2, 3, 8))
    u = torch.zeros((3, 8))
    for bad in (torch.float64, torch.bfloat16):
        with pytest.raises(TypeError):
            mla.mla_merge_partials(u_parts, torch.zeros((2, 3), dtype=bad), u)
        with pytest.raises(TypeError):
            mla.mla_merge_partials(u_parts, torch.zeros((2, 3)), u, torch.zeros(3, dtype=bad))


@pytest.mark.parametrize("args,want", [
    ((16, 32, 48, 64, 0, 10, 512, 0), INVALID),        # R = 0
    ((16, 32, 48, 64, 2, -1, 512, 0), INVALID),        # rows < 0
    ((16, 32, 48, 64, 2, 10, 12, 0), INVALID),         # d_c not a multiple of 8
    ((16, 32, 48, 64, 2, 10, 0, 0), INVALID),          # d_c = 0
    ((16, 32, 48, 64, 2, 10, 512, 7), INVALID),        # dtype
    ((None, 32, 48, 64, 2, 10, 512, 0), INVALID),      # u_parts
    ((16, None, 48, 64, 2, 10, 512, 0), INVALID),      # lse_parts
    ((16, 32, None, 64, 2, 10, 512, 0), INVALID),      # u
    ((17, 32, 48, 64, 2, 10, 512, 0), INVALID),        # u_parts not 16-byte aligned
    ((16, 34, 48, 64, 2, 10, 512, 0), INVALID),        # lse_parts not 4-byte aligned
    ((16, 32, 48, 68, 2, 10, 512, 0), INVALID),        # lse not 16-byte aligned
    ((None, None, None, None, 3, 0, 512, 0), OK),      # rows = 0: nothing to do
])
def test_merge_rejects_bad_arguments(lib, args, want):
    u_parts, lse_parts, u, lse, R, rows, d_c, dt = args
    assert lib.mla_merge_partials(u_parts, lse_parts, u, lse, R, rows, d_c, dt, None) == want
