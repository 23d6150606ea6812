"""Seeded synthetic inputs for absorbed-MLA decode.

This module only draws numbers and lays them out: it holds none of the
attention arithmetic (no projection, rotation, softmax or contraction).  Both
the CUDA path and the CPU oracle consume what it returns, so the two never
share any other code.

Every tensor comes from its own PCG64 stream, ``default_rng([seed, tag])``,
so a tensor's values do not depend on the sizes of the others.  Draws are
float32 and are rounded once to the storage type (bf16 round-to-nearest-even,
or kept as fp32); the returned arrays hold exactly the values the GPU sees,
widened to float32.

Workload shapes follow the DeepSeek-V3 MLA layer described in "MLA deep
compression" (operatorworld.com, sections on the low-rank projection and on
decoupled RoPE): 128 heads, latent d_c = 512, RoPE key d_R = 64, 576 cached
values per token; head dims 128 as in "Attention-head anatomy" §5.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np

TILE_TOKENS = 64  # cache rows per decode tile


# ----------------------------------------------------------------------------
# storage-type rounding
# ----------------------------------------------------------------------------
def bf16_round(x: np.ndarray, inplace: bool = False) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); float32 out.

    Works on the bit pattern in uint32 arithmetic (finite values, infinities
    and the NaNs drawn here never carry out of 32 bits), in chunks to bound
    temporaries."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if not inplace:
        x = x.copy()
    b = x.reshape(-1).view(np.uint32)
    step = 1 << 24
    for i in range(0, b.size, step):
        c = b[i:i + step]
        lsb = (c >> 16) & 1
        c += np.uint32(0x7FFF)
        c += lsb
        c &= np.uint32(0xFFFF0000)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# workload description
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    s_q: int
    n_h: int
    d_model: int
    d_c: int
    d_h: int
    d_v: int
    d_R: int
    page_size: int
    dtype: str                       # "bf16" or "fp32"
    seqlens: Optional[tuple] = None  # fixed lengths; None -> drawn from len_range
    len_range: Optional[tuple] = None  # (lo, hi) inclusive, uniform integers
    block_table: str = "identity"    # "identity" | "permuted"
    outlier_frac: float = 0.0        # fraction of cached rows scaled by outlier_scale
    outlier_scale: float = 8.0
    full_pipeline: bool = False      # cache made from hidden states (h -> c, k^R)
    rope_base: float = 10000.0
    scale: Optional[float] = None    # softmax scale; None -> 1/sqrt(d_h + d_R)
    tail_fill: str = "random"        # rows past seqlen inside a page: random|nan|zero
    seed: int = 0

    @property
    def width(self) -> int:
        return self.d_c + self.d_R

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d_h + self.d_R)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


V3 = dict(n_h=128, d_model=7168, d_c=512, d_h=128, d_v=128, d_R=64, dtype="bf16",
          page_size=64)

# The five workloads the bench and the parity tests are built on.
CONFIGS = {
    "tiny": Workload(name="tiny", B=2, s_q=1, n_h=8, d_model=256, d_c=64, d_h=32, d_v=32,
                     d_R=16, page_size=128, dtype="fp32", seqlens=(128, 128),
                     full_pipeline=True, seed=0),
    "v3": Workload(name="v3", B=16, s_q=1, seqlens=(4096,) * 16,
                   scale=1.0 / math.sqrt(192.0), seed=1, **V3),
    "ragged": Workload(name="ragged", B=64, s_q=1, len_range=(512, 32768),
                       block_table="permuted", seed=2, **V3),
    "mtp": Workload(name="mtp", B=32, s_q=2, seqlens=(8192,) * 32, seed=3, **V3),
    "long": Workload(name="long", B=4, s_q=1, seqlens=(131072,) * 4, outlier_frac=0.01,
                     seed=4, **V3),
}


def config(name: str, **overrides) -> Workload:
    w = CONFIGS[name]
    return replace(w, **overrides) if overrides else w


# ----------------------------------------------------------------------------
# draws
# ----------------------------------------------------------------------------
_TAGS = {"seqlens": 1, "perm": 2, "cache": 3, "outlier": 4, "h_q": 5, "W_Q": 6,
         "W_QR": 7, "W_UK": 8, "W_UV": 9, "W_DKV": 10, "W_KR": 11, "h_ctx": 12, "tail": 13,
         "gqa_kv": 14, "gqa_kr": 15, "gqa_q": 16}


_BLOCK = 1 << 22  # elements per independently seeded block of a large tensor


def _rng(seed: int, tag: str, block: int = -1) -> np.random.Generator:
    key = [int(seed), _TAGS[tag]] + ([] if block < 0 else [int(block)])
    return np.random.default_rng(key)


def _fill_block(flat, k, seed, tag, std, dtype):
    view = flat[k * _BLOCK:(k + 1) * _BLOCK]
    _rng(seed, tag, k).standard_normal(out=view, dtype=np.float32)
    if std != 1.0:
        view *= np.float32(std)
    if dtype == "bf16":
        bf16_round(view, inplace=True)


def _normal(seed: int, tag: str, shape, std: float = 1.0, dtype: str = "fp32") -> np.ndarray:
    """N(0, std^2) draws, rounded to `dtype`.  Block k of the flattened tensor
    comes from stream default_rng([seed, tag, k]), so the values do not depend
    on how many threads fill the blocks."""
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1)
    nblk = (flat.size + _BLOCK - 1) // _BLOCK
    if nblk <= 1:
        for k in range(nblk):
            _fill_block(flat, k, seed, tag, std, dtype)
        return out
    import concurrent.futures as cf
    import os
    with cf.ThreadPoolExecutor(max_workers=min(nblk, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda k: _fill_block(flat, k, seed, tag, std, dtype), range(nblk)))
    return out


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round an array drawn in float32 to the storage type (in place)."""
    return bf16_round(x, inplace=True) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def draw_seqlens(w: Workload) -> np.ndarray:
    if w.seqlens is not None:
        s = np.asarray(w.seqlens, dtype=np.int32)
        assert s.shape == (w.B,)
        return s
    lo, hi = w.len_range
    return _rng(w.seed, "seqlens").integers(lo, hi + 1, size=w.B, dtype=np.int64).astype(np.int32)


def make_block_table(w: Workload, seqlens: np.ndarray):
    """Page ids per sequence.  Returns (block_table [B, max_pages] int32, num_pages).

    identity: sequence b owns pages [b*max_pages, (b+1)*max_pages).
    permuted: the sum over b of ceil(L_b / page) pages, shuffled by a seeded
    permutation; unused slots of the table hold -1.
    """
    pages = [(int(L) + w.page_size - 1) // w.page_size for L in seqlens]
    max_pages = max(pages) if pages else 0
    bt = np.full((w.B, max(max_pages, 1)), -1, dtype=np.int32)
    if w.block_table == "identity":
        for b in range(w.B):
            bt[b, :pages[b]] = b * max_pages + np.arange(pages[b], dtype=np.int32)
        num_pages = w.B * max_pages
    else:
        total = int(sum(pages))
        perm = _rng(w.seed, "perm").permutation(total).astype(np.int32)
        off = 0
        for b in range(w.B):
            bt[b, :pages[b]] = perm[off:off + pages[b]]
            off += pages[b]
        num_pages = total
    return bt, num_pages


def cache_row_ids(w: Workload, block_table: np.ndarray, b: int, L: int) -> np.ndarray:
    """Physical cache row of each logical position 0..L-1 of sequence b."""
    j = np.arange(L, dtype=np.int64)
    return block_table[b, j // w.page_size].astype(np.int64) * w.page_size + j % w.page_size


def draw(w: Workload, with_weights: bool = True) -> dict:
    """All inputs of one decode step of workload ``w``.

    Keys (float32 arrays hold values exact in the storage dtype):
      seqlens [B] int32, block_table [B, max_pages] int32, num_pages int,
      qpos [B, s_q] int32 (query positions L_b - s_q + r),
      cache [num_pages*page, d_c + d_R]  (rows = c^KV || k^R; absent if full_pipeline),
      h_q [B, s_q, d_model], W_Q [n_h, d_h, d_model], W_QR [n_h, d_R, d_model],
      W_UK [n_h, d_h, d_c], W_UV [n_h, d_v, d_c],
      full pipeline only: h_ctx [B, L, d_model], W_DKV [d_c, d_model], W_KR [d_R, d_model].

    The cached k^R of a non-pipeline workload is drawn directly as N(0, 1):
    RoPE rotates consecutive pairs, and a rotated isotropic Gaussian pair is
    again an isotropic Gaussian pair, so the direct draw has exactly the
    distribution of "an N(0,1) vector rotated at its position".
    """
    seqlens = draw_seqlens(w)
    bt, num_pages = make_block_table(w, seqlens)
    rows = num_pages * w.page_size
    out = dict(seqlens=seqlens, block_table=bt, num_pages=num_pages,
               qpos=(seqlens[:, None] - w.s_q + np.arange(w.s_q, dtype=np.int32)[None, :]).astype(np.int32))
    dt = w.dtype
    if w.full_pipeline:
        assert w.seqlens is not None and len(set(w.seqlens)) == 1
        L = int(w.seqlens[0])
        out["h_ctx"] = _normal(w.seed, "h_ctx", (w.B, L, w.d_model), 1.0, dt)
        out["W_DKV"] = _normal(w.seed, "W_DKV", (w.d_c, w.d_model), 1 / math.sqrt(w.d_model), dt)
        out["W_KR"] = _normal(w.seed, "W_KR", (w.d_R, w.d_model), 1 / math.sqrt(w.d_model), dt)
        # the query tokens are the last s_q tokens appended to the context
        out["h_q"] = np.ascontiguousarray(out["h_ctx"][:, L - w.s_q:, :])
    else:
        plain = w.outlier_frac == 0 and w.tail_fill == "random"
        cache = _normal(w.seed, "cache", (rows, w.width), 1.0, dt if plain else "fp32")
        if w.outlier_frac > 0:
            valid = np.concatenate([cache_row_ids(w, bt, b, int(seqlens[b])) for b in range(w.B)])
            k = max(1, int(round(w.outlier_frac * valid.size)))
            pick = _rng(w.seed, "outlier").choice(valid, size=k, replace=False)
            cache[pick] *= np.float32(w.outlier_scale)
        if w.tail_fill != "random":
            used = np.zeros(rows, dtype=bool)
            for b in range(w.B):
                used[cache_row_ids(w, bt, b, int(seqlens[b]))] = True
            cache[~used] = np.nan if w.tail_fill == "nan" else 0.0
        out["cache"] = cache if plain else _store(cache, dt)
        if with_weights:
            out["h_q"] = _normal(w.seed, "h_q", (w.B, w.s_q, w.d_model), 1.0, dt)
    if with_weights:
        fi = 1 / math.sqrt(w.d_model)
        out["W_Q"] = _normal(w.seed, "W_Q", (w.n_h, w.d_h, w.d_model), fi, dt)
        out["W_QR"] = _normal(w.seed, "W_QR", (w.n_h, w.d_R, w.d_model), fi, dt)
        out["W_UK"] = _normal(w.seed, "W_UK", (w.n_h, w.d_h, w.d_c), 1 / math.sqrt(w.d_c), dt)
        out["W_UV"] = _normal(w.seed, "W_UV", (w.n_h, w.d_v, w.d_c), 1 / math.sqrt(w.d_c), dt)
    return out


def random_q(w: Workload, seed_tag: int = 0) -> np.ndarray:
    """An absorbed query tensor [B, s_q, n_h, d_c + d_R] drawn directly.

    Used where the decode is checked on its own bf16 inputs rather than
    through query formation: the long-context stress workload and the
    invariance checks.  The latent part is N(0, 0.25) and the RoPE part
    N(0, 1), the spreads the V3-shaped projections of N(0, 1) hidden states
    give.
    """
    g = np.random.default_rng([w.seed, 100 + seed_tag])
    q = g.standard_normal(size=(w.B, w.s_q, w.n_h, w.width), dtype=np.float32)
    q[..., :w.d_c] *= np.float32(0.5)
    return _store(q, w.dtype)


def draw_gqa(w: Workload, n_g: int) -> dict:
    """Inputs of a decode on GQLA's GQA path: the per-group expanded cache
    kv [rows, n_g, d_h + d_v] (keys then values of each group, N(0, 1)), the
    shared RoPE keys k_rope [rows, d_R] (N(0, 1), the distribution of a
    rotated N(0, 1) vector), and q [B, s_q, n_h, d_h + d_R] (q^nope N(0, 1/4),
    q^R N(0, 1)), with the sequence lengths and block table of ``w``."""
    seqlens = draw_seqlens(w)
    bt, num_pages = make_block_table(w, seqlens)
    rows = num_pages * w.page_size
    kv = _normal(w.seed, "gqa_kv", (rows, n_g, w.d_h + w.d_v), 1.0, w.dtype)
    kr = _normal(w.seed, "gqa_kr", (rows, w.d_R), 1.0, w.dtype)
    q = _normal(w.seed, "gqa_q", (w.B, w.s_q, w.n_h, w.d_h + w.d_R), 1.0, "fp32")
    q[..., :w.d_h] *= np.float32(0.5)
    q = _store(q, w.dtype)
    return dict(seqlens=seqlens, block_table=bt, num_pages=num_pages, kv=kv, k_rope=kr, q=q)
