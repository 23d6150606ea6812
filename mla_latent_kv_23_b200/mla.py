"""ctypes binding of libmla (include/mla.h).

Argument marshalling only: every function here reads shapes off torch
tensors, packs pointers and sizes, and calls the C entry point of the same
name; all computation happens in the library's CUDA kernels.  There is no
fallback: if libmla.so is missing or a call fails, MLAError is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmla.so")

MLA_DTYPE_BF16 = 0
MLA_DTYPE_FP32 = 1
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_CUDA",
          4: "MLA_ERR_WORKSPACE_TOO_SMALL", 5: "MLA_ERR_DEVICE_CHECK"}
DEVFLAG_BAD_SEQLEN, DEVFLAG_BAD_PAGE, DEVFLAG_TIMEOUT, DEVFLAG_LAYOUT, DEVFLAG_RANGE = 1, 2, 4, 8, 16


class MLAError(RuntimeError):
    def __init__(self, what: str, status: int, flags: int = 0):
        self.status = status
        self.flags = flags
        super().__init__(f"{what}: {STATUS.get(status, status)}" + (f" (flags {flags:#x})" if flags else ""))


class DecodeParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("kv_cache", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
                ("u", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("B", ctypes.c_int), ("s_q", ctypes.c_int), ("n_h", ctypes.c_int),
                ("d_c", ctypes.c_int), ("d_R", ctypes.c_int), ("page_size", ctypes.c_int),
                ("max_pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("dtype", ctypes.c_int),
                ("num_splits", ctypes.c_int), ("u_fp32", ctypes.c_int)]


class GqaParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("kv", ctypes.c_void_p), ("k_rope", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("B", ctypes.c_int), ("s_q", ctypes.c_int), ("n_h", ctypes.c_int),
                ("n_g", ctypes.c_int), ("d_h", ctypes.c_int), ("d_v", ctypes.c_int),
                ("d_R", ctypes.c_int), ("page_size", ctypes.c_int),
                ("max_pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("dtype", ctypes.c_int),
                ("num_splits", ctypes.c_int), ("o_fp32", ctypes.c_int)]


_V, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_P = ctypes.POINTER(DecodeParams)
_PG = ctypes.POINTER(GqaParams)
SIGNATURES = {
    "mla_status_string": ([_I], ctypes.c_char_p),
    "mla_absorb_weights": ([_V, _V, _V, _I, _I, _I, _I, _I, _V], _I),
    "mla_projection_workspace_size": ([_I, _I, _I, _I, ctypes.POINTER(_S)], _I),
    "mla_form_query": ([_V, _V, _V, _V, _V, _I, _I, _I, _I, _I, _F, _I, _V, _S, _V], _I),
    "mla_form_query_fused": ([_V, _V, _V, _V, _V, _V, _I, _I, _I, _I, _I, _I, _F, _V, _S, _V], _I),
    "mla_append_latent": ([_V, _V, _V, _V, _V, _V, _I, _I, _I, _V, _I, _I, _I, _I, _F, _I, _V, _S,
                           _V], _I),
    "mla_fold_output_weights": ([_V, _V, _V, _I, _I, _I, _I, _I, _V], _I),
    "mla_output_projection": ([_V, _I, _V, _V, _I, _I, _I, _V, _S, _V], _I),
    "mla_decode_workspace_size": ([_P, ctypes.POINTER(_S)], _I),
    "mla_decode": ([_P, _V, _S, _V], _I),
    "mla_decode_plan": ([_P, _V, _S, _V], _I),
    "mla_decode_attend": ([_P, _V, _S, _V], _I),
    "mla_decode_combine": ([_P, _V, _S, _V], _I),
    "mla_decode_kernel_info": ([_P, ctypes.POINTER(_I), ctypes.POINTER(_I)], _I),
    "mla_decode_noalloc": ([_P, _V], _I),
    "mla_decode_step": ([_P, _V, _V, _I, _V, _S, _V], _I),
    "mla_decode_gqa_workspace_size": ([_PG, ctypes.POINTER(_S)], _I),
    "mla_decode_gqa": ([_PG, _V, _S, _V], _I),
    "mla_up_proj": ([_V, _V, _V, _I, _I, _I, _I, _I, _I, _V], _I),
    "mla_merge_partials": ([_V, _V, _V, _V, _I, _I, _I, _I, _V], _I),
    "mla_check_device_errors": ([_V, ctypes.POINTER(_I)], _I),
    "mla_selftest_wait": ([_I, _V], _I),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmla.so (raises MLAError-compatible RuntimeError if absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m mla_latent_kv_23_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != 0:
        raise MLAError(what, status)


# ----------------------------------------------------------------------------
# torch marshalling helpers
# ----------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return MLA_DTYPE_BF16
    if t.dtype == torch.float32:
        return MLA_DTYPE_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        # the library's kernels read and write device memory only; a host
        # pointer would fault on the GPU
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------
def mla_absorb_weights(W_UK, W_Q, W_QK, stream=None) -> None:
    n_h, d_h, d_c = W_UK.shape
    d_model = W_Q.shape[2]
    assert W_Q.shape == (n_h, d_h, d_model) and W_QK.shape == (n_h, d_c, d_model)
    _check(lib().mla_absorb_weights(_ptr(W_UK), _ptr(W_Q), _ptr(W_QK), n_h, d_h, d_c, d_model,
                                    _dtype_code(W_UK), _stream(stream)), "mla_absorb_weights")


def mla_projection_workspace_size(rows0: int, rows1: int, T: int, x_fp32_K: int = 0) -> int:
    n = _S(0)
    _check(lib().mla_projection_workspace_size(rows0, rows1, T, x_fp32_K, ctypes.byref(n)),
           "mla_projection_workspace_size")
    return n.value


def projection_workspace(rows0: int, rows1: int, T: int, device, x_fp32_K: int = 0):
    """A zeroed projection workspace (the calls leave it zero again)."""
    torch = _torch()
    n = mla_projection_workspace_size(rows0, rows1, T, x_fp32_K)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def _ws(ws):
    return (None, 0) if ws is None else (_ptr(ws), ws.numel() * ws.element_size())


def mla_form_query(h, W_QK, W_QR, pos, q, rope_base: float = 10000.0, workspace=None,
                   stream=None) -> None:
    """q [T, n_h, d_c + d_R] = [W_QK h || RoPE(W_QR h, pos)]; bf16 needs a
    projection workspace (one is made if none is given)."""
    T, d_model = h.shape
    n_h, d_c, _ = W_QK.shape
    d_R = W_QR.shape[1]
    assert q.shape == (T, n_h, d_c + d_R)
    if workspace is None and _dtype_code(h) == MLA_DTYPE_BF16:
        workspace = projection_workspace(n_h * d_c, n_h * d_R, T, h.device)
    wp, wn = _ws(workspace)
    _check(lib().mla_form_query(_ptr(h), _ptr(W_QK), _ptr(W_QR), _ptr(pos), _ptr(q), T, n_h,
                                d_model, d_c, d_R, float(rope_base), _dtype_code(h), wp, wn,
                                _stream(stream)), "mla_form_query")


def mla_form_query_fused(h, W_Q, W_UK, W_QR, pos, q, rope_base: float = 10000.0, workspace=None,
                         stream=None) -> None:
    """q = [W_UK^T (W_Q h) || RoPE(W_QR h, pos)] without a precomputed W_QK."""
    T, d_model = h.shape
    n_h, d_h, d_c = W_UK.shape
    d_R = W_QR.shape[1]
    assert W_Q.shape == (n_h, d_h, d_model) and q.shape == (T, n_h, d_c + d_R)
    if workspace is None:
        workspace = projection_workspace(n_h * d_h, n_h * d_R, T, h.device)
    wp, wn = _ws(workspace)
    _check(lib().mla_form_query_fused(_ptr(h), _ptr(W_Q), _ptr(W_UK), _ptr(W_QR), _ptr(pos),
                                      _ptr(q), T, n_h, d_h, d_model, d_c, d_R, float(rope_base),
                                      wp, wn, _stream(stream)), "mla_form_query_fused")


def mla_append_latent(h, W_DKV, W_KR, seq_ids, pos, block_table, kv_cache, page_size: int,
                      rope_base: float = 10000.0, workspace=None, stream=None) -> None:
    T, d_model = h.shape
    d_c, d_R = W_DKV.shape[0], W_KR.shape[0]
    rows, width = kv_cache.shape
    assert width == d_c + d_R and rows % page_size == 0
    if workspace is None and _dtype_code(h) == MLA_DTYPE_BF16:
        workspace = projection_workspace(d_c, d_R, T, h.device)
    wp, wn = _ws(workspace)
    _check(lib().mla_append_latent(_ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(seq_ids), _ptr(pos),
                                   _ptr(block_table), block_table.shape[1], page_size,
                                   rows // page_size, _ptr(kv_cache), T, d_model, d_c, d_R,
                                   float(rope_base), _dtype_code(h), wp, wn, _stream(stream)),
           "mla_append_latent")


def mla_fold_output_weights(W_O, W_UV, W_OUV, stream=None) -> None:
    """W_OUV [d_model, n_h * d_c] = W_O [d_model, n_h * d_v] . blockdiag(W_UV [n_h, d_v, d_c])."""
    n_h, d_v, d_c = W_UV.shape
    d_model = W_O.shape[0]
    assert W_O.shape == (d_model, n_h * d_v) and W_OUV.shape == (d_model, n_h * d_c)
    _check(lib().mla_fold_output_weights(_ptr(W_O), _ptr(W_UV), _ptr(W_OUV), n_h, d_v, d_c,
                                         d_model, _dtype_code(W_O), _stream(stream)),
           "mla_fold_output_weights")


def mla_output_projection(x, W, y, workspace=None, stream=None) -> None:
    """y [T, M] = x [T, K] . W [M, K]^T (W bf16; x bf16 or float32)."""
    T, K = x.shape
    M = W.shape[0]
    assert W.shape == (M, K) and y.shape == (T, M)
    f32 = _dtype_code(x) == MLA_DTYPE_FP32
    if workspace is None:
        workspace = projection_workspace(M, 0, T, x.device, K if f32 else 0)
    wp, wn = _ws(workspace)
    _check(lib().mla_output_projection(_ptr(x), _dtype_code(x), _ptr(W), _ptr(y), T, K, M, wp, wn,
                                       _stream(stream)), "mla_output_projection")


def decode_params(q, kv_cache, block_table, seqlens, u, lse, page_size: int, d_R: int,
                  softmax_scale: float, num_splits: int = 0) -> DecodeParams:
    """Pack mla_decode_params from tensors: q [B, s_q, n_h, d_c + d_R],
    kv_cache [num_pages * page_size, d_c + d_R], block_table [B, max_pages],
    seqlens [B], u [B, s_q, n_h, d_c] (same dtype as q, or float32),
    lse [B, s_q, n_h] float32 or None."""
    torch = _torch()
    B, s_q, n_h, W = q.shape
    if u.dtype != q.dtype and u.dtype != torch.float32:
        raise TypeError("u must have the dtype of q or be float32")
    if lse is not None and lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    d_c = W - d_R
    rows = kv_cache.shape[0]
    return DecodeParams(q=_ptr(q), kv_cache=_ptr(kv_cache), block_table=_ptr(block_table),
                        seqlens=_ptr(seqlens), u=_ptr(u), lse=_ptr(lse), B=B, s_q=s_q, n_h=n_h,
                        d_c=d_c, d_R=d_R, page_size=page_size,
                        max_pages_per_seq=block_table.shape[1] if block_table.dim() == 2 else 1,
                        num_pages=max(rows // page_size, 1), softmax_scale=float(softmax_scale),
                        dtype=_dtype_code(q), num_splits=num_splits,
                        u_fp32=int(u.dtype == torch.float32))


def mla_decode_workspace_size(p: DecodeParams) -> int:
    n = _S(0)
    _check(lib().mla_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)),
           "mla_decode_workspace_size")
    return n.value


def mla_decode_kernel_info(p: DecodeParams) -> tuple[int, int]:
    tc, nc = _I(0), _I(0)
    _check(lib().mla_decode_kernel_info(ctypes.byref(p), ctypes.byref(tc), ctypes.byref(nc)),
           "mla_decode_kernel_info")
    return tc.value, nc.value


def _stage(name: str, p: DecodeParams, workspace, stream) -> None:
    fn = getattr(lib(), name)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(fn(ctypes.byref(p), _ptr(workspace), nbytes, _stream(stream)), name)


def mla_decode(p: DecodeParams, workspace, stream=None) -> None:
    _stage("mla_decode", p, workspace, stream)


def mla_decode_plan(p: DecodeParams, workspace, stream=None) -> None:
    _stage("mla_decode_plan", p, workspace, stream)


def mla_decode_attend(p: DecodeParams, workspace, stream=None) -> None:
    _stage("mla_decode_attend", p, workspace, stream)


def mla_decode_combine(p: DecodeParams, workspace, stream=None) -> None:
    _stage("mla_decode_combine", p, workspace, stream)


def mla_decode_step(p: DecodeParams, W_UV, o, workspace, stream=None) -> None:
    """mla_decode then o = W_UV u with the combine fused into the
    up-projection (fp32 u, the DeepSeek-V3 shape): o [B * s_q, n_h, d_v]."""
    d_v = W_UV.shape[1]
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().mla_decode_step(ctypes.byref(p), _ptr(W_UV), _ptr(o), d_v, _ptr(workspace), nbytes,
                                 _stream(stream)), "mla_decode_step")


def mla_decode_noalloc(p: DecodeParams, stream=None) -> None:
    """mla_decode with the library's own fixed scratch array (no workspace
    argument, no allocation); see include/mla.h for its size limit."""
    _check(lib().mla_decode_noalloc(ctypes.byref(p), _stream(stream)), "mla_decode_noalloc")


def mla_up_proj(u, W_UV, o, stream=None) -> None:
    """o [T, n_h, d_v] = W_UV [n_h, d_v, d_c] . u [T, n_h, d_c]; o has W_UV's
    dtype, u that dtype or float32."""
    T, n_h, d_c = u.shape
    d_v = W_UV.shape[1]
    assert W_UV.shape == (n_h, d_v, d_c) and o.shape == (T, n_h, d_v)
    if o.dtype != W_UV.dtype:
        raise TypeError("o must have the dtype of W_UV")
    _check(lib().mla_up_proj(_ptr(u), _ptr(W_UV), _ptr(o), T, n_h, d_c, d_v, _dtype_code(u),
                             _dtype_code(W_UV), _stream(stream)), "mla_up_proj")


def mla_merge_partials(u_parts, lse_parts, u, lse=None, stream=None) -> None:
    """Merge R partial (u, lse) over pieces of the same rows' context:
    u_parts [R, ..., d_c], lse_parts [R, ...] fp32 -> u [..., d_c], lse [...]."""
    R = u_parts.shape[0]
    d_c = u_parts.shape[-1]
    rows = u.numel() // d_c
    assert u_parts.numel() == R * rows * d_c and lse_parts.numel() == R * rows
    assert u_parts.is_contiguous() and lse_parts.is_contiguous() and u.is_contiguous()
    assert u_parts.dtype == u.dtype and (lse is None or lse.numel() == rows)
    torch = _torch()
    # the kernel reads the statistics as fp32 words
    if lse_parts.dtype != torch.float32 or (lse is not None and lse.dtype != torch.float32):
        raise TypeError("lse_parts and lse must be float32")
    if lse is not None and not lse.is_contiguous():
        raise ValueError("lse must be contiguous")
    _check(lib().mla_merge_partials(_ptr(u_parts), _ptr(lse_parts), _ptr(u), _ptr(lse), R, rows,
                                    d_c, _dtype_code(u), _stream(stream)), "mla_merge_partials")


def mla_check_device_errors(stream=None) -> int:
    """Synchronize, then return the device flags (raises MLAError if any is set)."""
    f = _I(0)
    st = lib().mla_check_device_errors(_stream(stream), ctypes.byref(f))
    if st != 0:
        raise MLAError("mla_check_device_errors", st, f.value)
    return f.value


def mla_selftest_wait(arrive: bool, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see include/mla.h)."""
    _check(lib().mla_selftest_wait(1 if arrive else 0, _stream(stream)), "mla_selftest_wait")


def mla_status_string(status: int) -> str:
    return lib().mla_status_string(status).decode()


# ----------------------------------------------------------------------------
# convenience: allocate outputs + workspace and run one decode
# ----------------------------------------------------------------------------
def decode(q, kv_cache, block_table, seqlens, page_size: int, d_R: int, softmax_scale: float,
           num_splits: int = 0, with_lse: bool = True, stream=None, u_dtype=None):
    """Returns (u [B, s_q, n_h, d_c], lse [B, s_q, n_h] or None); u has
    u_dtype (default: float32, which keeps the weighted latent sum unrounded
    for the up-projection)."""
    torch = _torch()
    B, s_q, n_h, W = q.shape
    u = torch.empty((B, s_q, n_h, W - d_R), dtype=u_dtype or torch.float32, device=q.device)
    lse = torch.empty((B, s_q, n_h), dtype=torch.float32, device=q.device) if with_lse else None
    p = decode_params(q, kv_cache, block_table, seqlens, u, lse, page_size, d_R, softmax_scale,
                      num_splits)
    ws = torch.empty(max(mla_decode_workspace_size(p), 256), dtype=torch.uint8, device=q.device)
    mla_decode(p, ws, stream)
    return u, lse


def decode_gqa(q, kv, k_rope, block_table, seqlens, page_size: int, softmax_scale: float,
               num_splits: int = 0, o_dtype=None, with_lse: bool = True, stream=None):
    """GQLA's GQA path: q [B, s_q, n_h, d_h + d_R], kv [rows, n_g, d_h + d_v],
    k_rope [rows, d_R] -> (o [B, s_q, n_h, d_v], lse [B, s_q, n_h] or None)."""
    torch = _torch()
    B, s_q, n_h, Wq = q.shape
    rows, n_g, Wkv = kv.shape
    d_R = k_rope.shape[1]
    d_h = Wq - d_R
    d_v = Wkv - d_h
    o = torch.empty((B, s_q, n_h, d_v), dtype=o_dtype or torch.float32, device=q.device)
    lse = torch.empty((B, s_q, n_h), dtype=torch.float32, device=q.device) if with_lse else None
    p = GqaParams(q=_ptr(q), kv=_ptr(kv), k_rope=_ptr(k_rope), block_table=_ptr(block_table),
                  seqlens=_ptr(seqlens), o=_ptr(o), lse=_ptr(lse), B=B, s_q=s_q, n_h=n_h, n_g=n_g,
                  d_h=d_h, d_v=d_v, d_R=d_R, page_size=page_size,
                  max_pages_per_seq=block_table.shape[1], num_pages=max(rows // page_size, 1),
                  softmax_scale=float(softmax_scale), dtype=_dtype_code(q), num_splits=num_splits,
                  o_fp32=int(o.dtype == torch.float32))
    n = _S(0)
    _check(lib().mla_decode_gqa_workspace_size(ctypes.byref(p), ctypes.byref(n)),
           "mla_decode_gqa_workspace_size")
    ws = torch.empty(max(n.value, 256), dtype=torch.uint8, device=q.device)
    _check(lib().mla_decode_gqa(ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream)),
           "mla_decode_gqa")
    return o, lse


def default_scale(d_h: int, d_R: int) -> float:
    return 1.0 / math.sqrt(d_h + d_R)
