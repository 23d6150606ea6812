"""The projections around the attention on the tensor cores, at the
DeepSeek-V3 shape (d_model = 7168, n_h = 128, d_h = d_v = 128, d_c = 512,
d_R = 64), against the fp64 oracle:

* query formation with the absorption done on the fly (W^UK^T (W^Q h), no
  W^QK) and with the offline W^QK ("MLA deep compression", absorption
  section, score equation; decoupled-RoPE section);
* the latent append c = W^DKV h, k^R = RoPE(W^KR h) written through a
  permuted block table (low-rank projection and decoupled-RoPE sections);
* the output side with W^UV folded into W^O offline, projecting u straight to
  the hidden size ("Attention-head anatomy" section 5), against the unfolded
  W^O (W^UV u)."""
import numpy as np
import pytest
import torch

from gpu_pipeline import ATOL_REL, f64, to_dev, to_dev_i32
from mla_latent_kv_23_b200 import mla, synth
from oracle import mla_oracle as orc

pytestmark = pytest.mark.gpu


def v3_proj(B, s_q=1, seqlens=None, **kw):
    seqlens = seqlens or tuple(int(x) for x in np.linspace(700, 9000, B))
    base = dict(name="v3-proj", B=B, s_q=s_q, n_h=128, d_model=7168, d_c=512, d_h=128, d_v=128,
                d_R=64, page_size=64, dtype="bf16", seqlens=seqlens, block_table="permuted",
                scale=1 / np.sqrt(192.0), seed=41)
    base.update(kw)
    return synth.Workload(**base)


def rel_err(got, ref):
    return float(np.max(np.abs(got - ref) / (1 + np.abs(ref))))


@pytest.mark.parametrize("B,s_q", [(16, 1), (40, 2)])
def test_fused_query_formation(B, s_q):
    # 16 and 80 query rows (more than one 64-row launch), every head and value
    w = v3_proj(B, s_q)
    inp = synth.draw(w)
    T = w.B * w.s_q
    h = to_dev(inp["h_q"].reshape(T, w.d_model), w)
    pos = to_dev_i32(inp["qpos"].reshape(-1))
    W_Q, W_UK, W_QR = (to_dev(inp[k], w) for k in ("W_Q", "W_UK", "W_QR"))
    q = torch.full((T, w.n_h, w.width), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = mla.projection_workspace(w.n_h * w.d_h, w.n_h * w.d_R, T, "cuda")
    mla.mla_form_query_fused(h, W_Q, W_UK, W_QR, pos, q, rope_base=w.rope_base, workspace=ws)
    # a second call on the same workspace (left zero by the first)
    q2 = torch.empty_like(q)
    mla.mla_form_query_fused(h, W_Q, W_UK, W_QR, pos, q2, rope_base=w.rope_base, workspace=ws)
    mla.mla_check_device_errors()
    assert torch.equal(q, q2)
    assert int(torch.count_nonzero(ws)) == 0
    ref = orc.absorbed_queries_all(inp, w).reshape(T, w.n_h, w.width)
    got = f64(q)
    assert np.isfinite(got).all()
    assert rel_err(got[..., :w.d_c], ref[..., :w.d_c]) <= ATOL_REL
    assert rel_err(got[..., w.d_c:], ref[..., w.d_c:]) <= ATOL_REL


def test_absorbed_query_formation_on_tensor_cores():
    # the offline W^QK path (bf16 on the tensor cores) agrees with the same
    # oracle queries
    w = v3_proj(8, d_model=1024)
    inp = synth.draw(w)
    from gpu_pipeline import absorb_and_query
    q, _ = absorb_and_query(w, inp)
    ref = orc.absorbed_queries_all(inp, w)
    assert rel_err(f64(q), ref) <= ATOL_REL


def test_latent_append_at_the_v3_shape():
    # 50 new tokens of 3 sequences at scattered positions of a permuted paged
    # cache; the written rows are [W^DKV h || RoPE(W^KR h, pos)], every other
    # row keeps its contents
    w = v3_proj(3, seqlens=(1000, 4097, 300))
    inp = synth.draw(w)
    rng = np.random.default_rng(6)
    seq = rng.integers(0, w.B, size=50).astype(np.int32)
    pos = np.array([rng.integers(0, int(inp["seqlens"][b])) for b in seq], np.int32)
    # distinct target rows
    _, keep = np.unique(seq.astype(np.int64) * 100000 + pos, return_index=True)
    seq, pos = seq[np.sort(keep)], pos[np.sort(keep)]
    T = len(seq)
    h = synth._normal(w.seed, "h_ctx", (T, w.d_model), 1.0, "bf16")
    W_DKV = synth._normal(w.seed, "W_DKV", (w.d_c, w.d_model), 1 / np.sqrt(w.d_model), "bf16")
    W_KR = synth._normal(w.seed, "W_KR", (w.d_R, w.d_model), 1 / np.sqrt(w.d_model), "bf16")
    cache = to_dev(inp["cache"], w)
    before = cache.clone()
    bt = to_dev_i32(inp["block_table"])
    mla.mla_append_latent(to_dev(h, w), to_dev(W_DKV, w), to_dev(W_KR, w), to_dev_i32(seq),
                          to_dev_i32(pos), bt, cache, w.page_size, rope_base=w.rope_base)
    mla.mla_check_device_errors()
    rows = np.array([synth.cache_row_ids(w, inp["block_table"], int(b), int(p) + 1)[-1]
                     for b, p in zip(seq, pos)])
    got = f64(cache)[rows]
    c_ref = orc.latent(W_DKV, h)
    kr_ref = orc.rope_key(W_KR, h, pos, w.rope_base)
    assert rel_err(got[:, :w.d_c], c_ref) <= ATOL_REL
    assert rel_err(got[:, w.d_c:], kr_ref) <= ATOL_REL
    mask = torch.ones(cache.shape[0], dtype=torch.bool, device="cuda")
    mask[torch.from_numpy(rows).cuda()] = False
    assert torch.equal(cache[mask], before[mask])


def test_output_side_folded_into_w_o():
    # y = W^OUV u (u fp32 from the decode, folded weights) against the
    # definition y = W^O concat_i(W^UV_i u_i); and against the unfolded path
    # on the GPU (mla_up_proj then the output projection with W^O)
    n_h, d_v, d_c, d_model, T = 128, 128, 512, 7168, 8
    g = np.random.default_rng(12)
    W_UV = synth.bf16_round((g.standard_normal((n_h, d_v, d_c)) / np.sqrt(d_c)).astype(np.float32))
    W_O = synth.bf16_round((g.standard_normal((d_model, n_h * d_v)) / np.sqrt(n_h * d_v))
                           .astype(np.float32))
    u = (g.standard_normal((T, n_h, d_c)) * 3).astype(np.float32)
    dW_UV = torch.from_numpy(W_UV).cuda().to(torch.bfloat16)
    dW_O = torch.from_numpy(W_O).cuda().to(torch.bfloat16)
    W_OUV = torch.empty((d_model, n_h * d_c), dtype=torch.bfloat16, device="cuda")
    mla.mla_fold_output_weights(dW_O, dW_UV, W_OUV)
    du = torch.from_numpy(u).cuda()
    y = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    mla.mla_output_projection(du.view(T, n_h * d_c), W_OUV, y)
    o = torch.empty((T, n_h, d_v), dtype=torch.bfloat16, device="cuda")
    mla.mla_up_proj(du, dW_UV, o)
    y2 = torch.empty_like(y)
    mla.mla_output_projection(o.view(T, n_h * d_v), dW_O, y2)
    mla.mla_check_device_errors()
    ref = orc.output_projection(orc.up_project(u, W_UV), W_O)
    assert rel_err(f64(y), ref) <= ATOL_REL
    assert rel_err(f64(y2), ref) <= ATOL_REL
    # the folded weights themselves
    Wf = f64(W_OUV)
    for i in (0, 77, 127):
        blk = W_O.astype(np.float64)[:, i * d_v:(i + 1) * d_v] @ W_UV[i].astype(np.float64)
        assert rel_err(Wf[:, i * d_c:(i + 1) * d_c], blk) <= 2.0 ** -7
