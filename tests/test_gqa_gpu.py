"""GQLA's GQA path on the tensor cores (GQLA summary, abstract and method
paragraphs): decode over a per-group expanded cache with s_q = 1 and 2, at a
LLaMA-3-8B-like grouping (32 query heads, 8 groups, d_h = d_v = 128, a
64-wide shared RoPE key), against the oracle's GQA decode for every
(sequence, query row, head)."""
import numpy as np
import pytest
import torch

from gpu_pipeline import ATOL_REL, f64, lse_err, to_dev, to_dev_i32
from mla_latent_kv_23_b200 import mla, synth
from oracle import mla_oracle as orc

pytestmark = pytest.mark.gpu


def gqa_workload(s_q, seqlens, n_h=32):
    return synth.Workload(name="gqla", B=len(seqlens), s_q=s_q, n_h=n_h, d_model=256, d_c=512,
                          d_h=128, d_v=128, d_R=64, page_size=64, dtype="bf16", seqlens=seqlens,
                          block_table="permuted", scale=1 / np.sqrt(192.0), seed=51)


@pytest.mark.parametrize("s_q,splits", [(2, 0), (2, 7), (1, 0), (1, 5)])
def test_gqa_decode_all_rows(s_q, splits):
    n_g = 8
    w = gqa_workload(s_q, (700, 65, 2, 3000, 1025))
    inp = synth.draw_gqa(w, n_g)
    q, kv, kr = to_dev(inp["q"], w), to_dev(inp["kv"], w), to_dev(inp["k_rope"], w)
    bt, sl = to_dev_i32(inp["block_table"]), to_dev_i32(inp["seqlens"])
    o, lse = mla.decode_gqa(q, kv, kr, bt, sl, w.page_size, w.softmax_scale, num_splits=splits)
    mla.mla_check_device_errors()
    ref = orc.decode_gqa(inp["q"], inp["kv"], inp["k_rope"], inp["block_table"], inp["seqlens"],
                         w, n_g)
    oo, ll = f64(o), f64(lse)
    worst_o = worst_l = 0.0
    for (b, r, i), (o_ref, lse_ref) in ref.items():
        worst_o = max(worst_o, float(np.max(np.abs(oo[b, r, i] - o_ref) / (1 + np.abs(o_ref)))))
        worst_l = max(worst_l, lse_err(ll[b, r, i], lse_ref))
    print(f"gqa s_q={s_q} splits={splits}: o {worst_o:.2e} lse {worst_l:.3f}")
    assert len(ref) == w.B * w.s_q * w.n_h
    assert worst_o <= ATOL_REL and worst_l <= 1.0


def test_gqa_two_rows_share_the_reads_and_row0_matches_one_row():
    # row 0 of an s_q = 2 decode sees the same positions as an s_q = 1 decode
    # of the context one shorter
    n_g = 4
    w2 = gqa_workload(2, (300, 1025, 64), n_h=16)
    inp = synth.draw_gqa(w2, n_g)
    q, kv, kr = to_dev(inp["q"], w2), to_dev(inp["kv"], w2), to_dev(inp["k_rope"], w2)
    bt = to_dev_i32(inp["block_table"])
    o2, l2 = mla.decode_gqa(q, kv, kr, bt, to_dev_i32(inp["seqlens"]), w2.page_size,
                            w2.softmax_scale, num_splits=1)
    o1, l1 = mla.decode_gqa(q[:, :1].contiguous(), kv, kr, bt, to_dev_i32(inp["seqlens"] - 1),
                            w2.page_size, w2.softmax_scale, num_splits=1)
    mla.mla_check_device_errors()
    assert torch.allclose(o1[:, 0], o2[:, 0], rtol=0, atol=1e-6)
    assert torch.allclose(l1[:, 0], l2[:, 0], rtol=0, atol=1e-6)
