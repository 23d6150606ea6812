"""Pins for the CPU oracle: each check ties it to something other than itself.

* brute force: a separate triple-loop implementation in plain Python floats;
* the associativity identity the pages derive (absorbed == expanded);
* closed forms: uniform scores, a single cached token, a dominant token;
* library special cases: scipy's logsumexp / softmax;
* RoPE closed forms and its relative-position property;
* the cache-size figures the pages print (tests/golden/kv_cache_figures.json);
* invariants: block-table permutation, causal row 0 == shorter context.

The last group plants plausible mistakes into the oracle (on the CPU) and
checks that the pins above catch each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from brute_force import brute_decode
from mla_latent_kv_23_b200 import synth
from oracle import mla_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_cache_figures.json")


def tiny_workload(**kw):
    base = dict(name="bf", B=2, s_q=1, n_h=2, d_model=6, d_c=4, d_h=3, d_v=2, d_R=4,
                page_size=2, dtype="fp32", seqlens=(3, 5), block_table="permuted", seed=11)
    base.update(kw)
    return synth.Workload(**base)


def _max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def compare_to_brute(w, inp, tol=1e-12):
    ref = brute_decode(inp, w)
    got = orc.decode_expanded(inp, w)
    worst = 0.0
    for key, (o_bf, lse_bf) in ref.items():
        o, lse = got[key]
        worst = max(worst, _max_abs(o, o_bf), abs(lse - lse_bf))
    return worst


# ----------------------------------------------------------------------------
# brute force
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("s_q", [1, 2])
@pytest.mark.parametrize("seqlens", [(1, 2), (3, 5), (5, 4)])
def test_oracle_matches_brute_force_paged(s_q, seqlens):
    if s_q > min(seqlens):
        pytest.skip("L >= s_q required")
    w = tiny_workload(s_q=s_q, seqlens=seqlens)
    inp = synth.draw(w)
    assert compare_to_brute(w, inp) < 1e-12


@pytest.mark.parametrize("s_q", [1, 2])
def test_oracle_matches_brute_force_full_pipeline(s_q):
    # h -> c, k^R = RoPE(W^KR h, t) -> cache; queries are the last tokens.
    w = tiny_workload(s_q=s_q, seqlens=(5, 5), full_pipeline=True, block_table="identity",
                      page_size=4)
    inp = synth.draw(w)
    assert compare_to_brute(w, inp) < 1e-12


def test_tiny_config_brute_force_sample():
    # the tiny workload itself, restricted to 2 heads and 9 cached tokens
    w = synth.config("tiny").with_(n_h=2, seqlens=(9, 9), page_size=64)
    inp = synth.draw(w)
    assert compare_to_brute(w, inp) < 1e-12


# ----------------------------------------------------------------------------
# associativity: absorbed == expanded
# ----------------------------------------------------------------------------
def medium_workload(**kw):
    base = dict(name="med", B=3, s_q=2, n_h=4, d_model=24, d_c=16, d_h=8, d_v=8, d_R=8,
                page_size=8, dtype="bf16", seqlens=(37, 9, 64), block_table="permuted", seed=5)
    base.update(kw)
    return synth.Workload(**base)


def _absorbed_q(inp, w, W_QK=None):
    q = np.zeros((w.B, w.s_q, w.n_h, w.width))
    for b in range(w.B):
        for r in range(w.s_q):
            for i in range(w.n_h):
                q[b, r, i] = orc.absorbed_query(inp, w, b, r, i,
                                                None if W_QK is None else W_QK[i])
    return q


@pytest.mark.parametrize("use_wqk", [False, True])
def test_absorbed_equals_expanded(use_wqk):
    w = medium_workload()
    inp = synth.draw(w)
    W_QK = orc.absorb_weights(inp["W_UK"], inp["W_Q"]) if use_wqk else None
    q = _absorbed_q(inp, w, W_QK)
    ua = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w)
    ex = orc.decode_expanded(inp, w)
    for key, (o, lse) in ex.items():
        u, lse_a = ua[key]
        o_from_u = orc.up_project(u[None, :], inp["W_UV"][key[2]][None])[0]
        assert _max_abs(o_from_u, o) < 1e-10
        assert abs(lse_a - lse) < 1e-10


@pytest.mark.parametrize("s_q", [1, 2])
def test_all_heads_helpers_reproduce_the_expanded_definition(s_q):
    # absorbed_queries + decode_absorbed_seq (all heads of a sequence as matrix
    # products) must give the expanded oracle's o and lse through o = W^UV u
    w = medium_workload(s_q=s_q)
    inp = synth.draw(w)
    ex = orc.decode_expanded(inp, w)
    for b in range(w.B):
        q_b = np.stack([orc.absorbed_queries(inp, w, b, r) for r in range(w.s_q)])
        u, lse, abs_c = orc.decode_absorbed_seq(q_b, inp["cache"], inp["block_table"],
                                                int(inp["seqlens"][b]), b, w, want_abs=True)
        for r in range(w.s_q):
            o = orc.up_project(u[r], inp["W_UV"])
            for i in range(w.n_h):
                o_ref, lse_ref = ex[(b, r, i)]
                assert _max_abs(o[i], o_ref) < 1e-10
                assert abs(lse[r, i] - lse_ref) < 1e-10
        # the weighted absolute sum bounds |u| and is u itself when every
        # latent is non-negative
        assert np.all(abs_c >= np.abs(u) - 1e-12)
    cache = np.abs(inp["cache"])
    b = 0
    q_b = np.stack([orc.absorbed_queries(inp, w, b, r) for r in range(w.s_q)])
    u, _, abs_c = orc.decode_absorbed_seq(q_b, cache, inp["block_table"], int(inp["seqlens"][b]),
                                          b, w, want_abs=True)
    assert _max_abs(abs_c, u) < 1e-12


def test_batched_queries_reproduce_the_expanded_definition():
    # absorbed_queries_all (all rows at once) through the absorbed decode
    # gives the expanded oracle's o and lse
    w = medium_workload()
    inp = synth.draw(w)
    qa = orc.absorbed_queries_all(inp, w)
    ua = orc.decode_absorbed(qa, inp["cache"], inp["block_table"], inp["seqlens"], w)
    for key, (o, lse) in orc.decode_expanded(inp, w).items():
        u, lse_a = ua[key]
        assert _max_abs(orc.up_project(u[None, :], inp["W_UV"][key[2]][None])[0], o) < 1e-10
        assert abs(lse_a - lse) < 1e-10


def test_output_projection_brute_force():
    # y_t[m] = sum over heads i and value dims v of W_O[m, i d_v + v] o_t[i, v],
    # summed term by term with math.fsum
    rng = np.random.default_rng(8)
    T, n_h, d_v, d_model = 3, 4, 5, 7
    o = rng.standard_normal((T, n_h, d_v))
    W_O = rng.standard_normal((d_model, n_h * d_v))
    y = orc.output_projection(o, W_O)
    for t in range(T):
        for m in range(d_model):
            ref = math.fsum(W_O[m, i * d_v + v] * o[t, i, v] for i in range(n_h) for v in range(d_v))
            assert abs(y[t, m] - ref) < 1e-12 * (1 + abs(ref))
    # heads are concatenated in order: moving one head's values moves the
    # contribution to that head's columns of W_O only
    o2 = o.copy()
    o2[:, 1] = 0.0
    W2 = W_O.copy()
    W2[:, d_v:2 * d_v] = 0.0
    assert _max_abs(orc.output_projection(o2, W_O), orc.output_projection(o, W2)) < 1e-12


def test_absorbed_scores_equal_expanded_scores():
    rng = np.random.default_rng(3)
    n_h, d_h, d_c, d_model = 3, 5, 7, 11
    W_UK = rng.standard_normal((n_h, d_h, d_c))
    W_Q = rng.standard_normal((n_h, d_h, d_model))
    h = rng.standard_normal(d_model)
    c = rng.standard_normal(d_c)
    W_QK = orc.absorb_weights(W_UK, W_Q)
    for i in range(n_h):
        lhs = (W_QK[i] @ h) @ c
        rhs = (W_Q[i] @ h) @ (W_UK[i] @ c)
        assert abs(lhs - rhs) < 1e-12 * (1 + abs(rhs))


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------
def test_uniform_scores_give_mean_of_values():
    w = medium_workload(s_q=1)
    inp = synth.draw(w)
    inp["W_Q"] = np.zeros_like(inp["W_Q"])
    inp["W_QR"] = np.zeros_like(inp["W_QR"])
    out = orc.decode_expanded(inp, w)
    for (b, r, i), (o, lse) in out.items():
        L = int(inp["seqlens"][b])
        rows = orc.gather_rows(inp["cache"], inp["block_table"], w.page_size, b, L)
        mean_c = rows[:, :w.d_c].mean(axis=0)
        assert _max_abs(o, np.asarray(inp["W_UV"][i], np.float64) @ mean_c) < 1e-12
        assert abs(lse - math.log(L)) < 1e-12


def test_single_token_returns_its_value():
    w = medium_workload(s_q=1, seqlens=(1, 1, 1))
    inp = synth.draw(w)
    out = orc.decode_expanded(inp, w)
    for (b, r, i), (o, lse) in out.items():
        row = orc.gather_rows(inp["cache"], inp["block_table"], w.page_size, b, 1)[0]
        assert _max_abs(o, np.asarray(inp["W_UV"][i], np.float64) @ row[:w.d_c]) < 1e-12
        q = orc.query_head(inp["W_Q"][i], inp["W_QR"][i], inp["h_q"][b, 0], 0, w.rope_base)
        k = np.concatenate([np.asarray(inp["W_UK"][i], np.float64) @ row[:w.d_c], row[w.d_c:]])
        assert abs(lse - w.softmax_scale * float(q @ k)) < 1e-12


def test_dominant_token():
    rng = np.random.default_rng(9)
    L, d, dv, scale = 40, 12, 5, 0.25
    q = rng.standard_normal(d)
    K = np.zeros((L, d))
    K[17] = q * (60.0 / (scale * float(q @ q)))      # score of row 17 = 60, others 0
    V = rng.standard_normal((L, dv))
    o, lse, a = orc.softmax_attend(q, K, V, scale, L)
    assert abs(lse - (60.0 + math.log1p((L - 1) * math.exp(-60.0)))) < 1e-12
    # all other rows carry weight e^-60 / (1 + (L-1) e^-60) each
    assert _max_abs(o, V[17]) <= 2 * L * math.exp(-60.0) * np.abs(V).max()


def test_softmax_matches_scipy():
    rng = np.random.default_rng(4)
    q = rng.standard_normal(10)
    K = rng.standard_normal((33, 10)) * 3
    V = rng.standard_normal((33, 4))
    o, lse, a = orc.softmax_attend(q, K, V, 0.7, 29)
    s = 0.7 * (K[:29] @ q)
    assert abs(lse - scipy.special.logsumexp(s)) < 1e-12
    assert _max_abs(a, scipy.special.softmax(s)) < 1e-15
    assert _max_abs(o, scipy.special.softmax(s) @ V[:29]) < 1e-12


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------
def test_rope_two_dims_is_rotation_by_pos_radians():
    x = np.array([0.3, -1.2])
    for pos in [0, 1, 7, 1000]:
        c, s = math.cos(pos), math.sin(pos)
        want = [0.3 * c + 1.2 * s, 0.3 * s - 1.2 * c]
        assert _max_abs(orc.rope(x, pos, 10000.0), want) < 1e-12


def test_rope_four_dims_second_pair_uses_base_power():
    x = np.array([1.0, 0.0, 0.0, 1.0])
    pos = 3
    th1 = 10000.0 ** (-2.0 / 4.0)               # 0.01
    want = [math.cos(3), math.sin(3), -math.sin(3 * th1), math.cos(3 * th1)]
    assert abs(th1 - 0.01) < 1e-15
    assert _max_abs(orc.rope(x, pos, 10000.0), want) < 1e-12


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    base = 10000.0
    d1 = orc.rope(q, 100, base) @ orc.rope(k, 37, base)
    d2 = orc.rope(q, 100 + 4321, base) @ orc.rope(k, 37 + 4321, base)
    assert abs(d1 - d2) < 1e-9
    assert abs(np.linalg.norm(orc.rope(q, 77, base)) - np.linalg.norm(q)) < 1e-12
    assert _max_abs(orc.rope(q, 0, base), q) == 0.0


# ----------------------------------------------------------------------------
# figures the pages print
# ----------------------------------------------------------------------------
def test_printed_cache_figures():
    g = json.load(open(GOLDEN))
    for e in g["kv_bytes"]:
        assert orc.kv_bytes_per_token(e["layers"], e["kv_heads"], e["head_dim"], e["bytes"]) == e["expected"], e["what"]
    for e in g["context_bytes"]:
        assert e["per_token_bytes"] * e["tokens"] * e["sequences"] == e["expected"], e["what"]
        assert orc.kv_bytes_per_token(32, 32, 128, 2) == e["per_token_bytes"]
    m = {e["what"]: e for e in g["mla"]}
    e = m["K/V values per token per layer in DeepSeek-V3 before MLA"]
    assert orc.mha_kv_elems(e["n_h"], e["d_h"]) == e["expected"]
    e = m["MLA cached values per token per layer"]
    assert orc.mla_cache_elems(e["d_c"], e["d_R"]) == e["expected"]
    e = m["DeepSeek-V2 cache per token, 60 layers, 16-bit"]
    assert orc.mla_cache_elems(e["d_c"], e["d_R"]) * e["layers"] * e["bytes"] == e["expected"]
    assert e["expected"] / 1024 == 67.5
    e = m["MLA cache expressed as GQA groups of K and V heads of dim 128"]
    assert 2 * e["groups"] * e["head_dim"] == e["expected"] == orc.mla_cache_elems(512, 64)
    e = m["GQLA absorbed-path cache as a fraction of the LLaMA-3-8B GQA cache (8 KV heads of 128)"]
    frac = orc.mla_cache_elems(e["d_c"], e["d_R"]) / orc.mha_kv_elems(e["kv_heads"], e["head_dim"])
    assert frac == e["expected_fraction"]


def test_workload_cache_width_is_576():
    for name in ["v3", "ragged", "mtp", "long"]:
        w = synth.config(name)
        assert w.width == orc.mla_cache_elems(w.d_c, w.d_R) == 576
    assert synth.config("tiny").width == 80


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------
def test_block_table_permutation_invariance():
    w = medium_workload(block_table="identity", s_q=1)
    inp = synth.draw(w)
    rng = np.random.default_rng(1)
    perm = rng.permutation(inp["num_pages"])           # new page id of old page p
    cache2 = np.empty_like(inp["cache"])
    P = w.page_size
    for p in range(inp["num_pages"]):
        cache2[perm[p] * P:(perm[p] + 1) * P] = inp["cache"][p * P:(p + 1) * P]
    bt2 = np.where(inp["block_table"] >= 0, perm[np.maximum(inp["block_table"], 0)], -1)
    inp2 = dict(inp, cache=cache2, block_table=bt2.astype(np.int32))
    a, b = orc.decode_expanded(inp, w), orc.decode_expanded(inp2, w)
    for key in a:
        assert np.array_equal(a[key][0], b[key][0]) and a[key][1] == b[key][1]


def test_causal_row0_equals_shorter_context():
    w = medium_workload(s_q=2)
    inp = synth.draw(w)
    two = orc.decode_expanded(inp, w)
    w1 = w.with_(s_q=1)
    inp1 = dict(inp, seqlens=inp["seqlens"] - 1, h_q=inp["h_q"][:, :1],
                qpos=inp["qpos"][:, :1])
    one = orc.decode_expanded(inp1, w1)
    for (b, r, i), (o, lse) in one.items():
        o2, lse2 = two[(b, 0, i)]
        assert _max_abs(o, o2) == 0.0 and lse == lse2


# ----------------------------------------------------------------------------
# the pins catch planted mistakes
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mistake", ["rope_sign", "drop_rope_term", "mask_off_by_one",
                                     "transpose_uk", "scale_missing"])
def test_pins_catch_planted_mistakes(monkeypatch, mistake):
    w = tiny_workload(s_q=2, seqlens=(4, 5))
    inp = synth.draw(w)
    assert compare_to_brute(w, inp) < 1e-12
    if mistake == "rope_sign":
        orig = orc.rope
        monkeypatch.setattr(orc, "rope", lambda x, pos, base: orig(x, -np.asarray(pos), base))
    elif mistake == "drop_rope_term":
        orig = orc.expanded_kv
        monkeypatch.setattr(orc, "expanded_kv",
                            lambda C, KR, a, b: orig(C, np.zeros_like(np.asarray(KR, float)), a, b))
    elif mistake == "mask_off_by_one":
        orig = orc.softmax_attend
        monkeypatch.setattr(orc, "softmax_attend",
                            lambda q, K, V, s, n_valid: orig(q, K, V, s, max(1, n_valid - 1)))
    elif mistake == "transpose_uk":
        orig = orc.expanded_kv
        monkeypatch.setattr(orc, "expanded_kv",
                            lambda C, KR, a, b: orig(C, KR, np.asarray(a)[::-1], b))
    elif mistake == "scale_missing":
        orig = orc.softmax_attend
        monkeypatch.setattr(orc, "softmax_attend", lambda q, K, V, s, n_valid: orig(q, K, V, 1.0, n_valid))
    assert compare_to_brute(w, inp) > 1e-6


# ----------------------------------------------------------------------------
# GQLA's GQA path
# ----------------------------------------------------------------------------
def test_gqa_decode_brute_force():
    w = synth.Workload(name="gqa-bf", B=2, s_q=2, n_h=4, d_model=6, d_c=8, d_h=3, d_v=2, d_R=2,
                       page_size=2, dtype="fp32", seqlens=(3, 5), block_table="permuted", seed=13)
    inp = synth.draw_gqa(w, n_g=2)
    ref = orc.decode_gqa(inp["q"], inp["kv"], inp["k_rope"], inp["block_table"], inp["seqlens"], w, 2)
    for (b, r, i), (o, lse) in ref.items():
        g = i // 2
        L = int(inp["seqlens"][b])
        rid = synth.cache_row_ids(w, inp["block_table"], b, L)
        scores = []
        for j in range(L - w.s_q + r + 1):
            row = rid[j]
            dot = math.fsum([float(inp["q"][b, r, i, k]) * float(inp["kv"][row, g, k]) for k in range(w.d_h)] +
                            [float(inp["q"][b, r, i, w.d_h + k]) * float(inp["k_rope"][row, k])
                             for k in range(w.d_R)])
            scores.append(w.softmax_scale * dot)
        mx = max(scores)
        ex = [math.exp(x - mx) for x in scores]
        z = math.fsum(ex)
        assert abs(lse - (mx + math.log(z))) < 1e-12
        for v in range(w.d_v):
            ref_v = math.fsum(ex[j] / z * float(inp["kv"][rid[j], g, w.d_h + v]) for j in range(len(ex)))
            assert abs(o[v] - ref_v) < 1e-12


def test_gqa_and_mla_paths_agree_with_tied_weights():
    # the two decoding paths over the same GQLA weights: heads of a group share
    # W^UK_g, W^UV_g; the GQA path on the expanded cache equals the MLA path
    # (expanded definition, and absorbed u with o = W^UV_g u)
    n_g = 2
    w = medium_workload(s_q=2)
    inp = synth.draw(w)
    hpg = w.n_h // n_g
    rng = np.random.default_rng(4)
    W_UK_g = rng.standard_normal((n_g, w.d_h, w.d_c)) / math.sqrt(w.d_c)
    W_UV_g = rng.standard_normal((n_g, w.d_v, w.d_c)) / math.sqrt(w.d_c)
    tied = dict(inp)
    tied["W_UK"] = np.repeat(W_UK_g, hpg, axis=0)
    tied["W_UV"] = np.repeat(W_UV_g, hpg, axis=0)
    mla_o = orc.decode_expanded(tied, w)
    kv, kr = orc.expand_gqa_cache(inp["cache"], W_UK_g, W_UV_g, w.d_c)
    q = np.zeros((w.B, w.s_q, w.n_h, w.d_h + w.d_R))
    for b in range(w.B):
        for r in range(w.s_q):
            for i in range(w.n_h):
                q[b, r, i] = orc.query_head(inp["W_Q"][i], inp["W_QR"][i], inp["h_q"][b, r],
                                            int(inp["qpos"][b, r]), w.rope_base)
    gqa = orc.decode_gqa(q, kv, kr, inp["block_table"], inp["seqlens"], w, n_g)
    qa = np.stack([np.stack([orc.absorbed_queries(tied, w, b, r) for r in range(w.s_q)])
                   for b in range(w.B)])
    ua = orc.decode_absorbed(qa, inp["cache"], inp["block_table"], inp["seqlens"], w)
    for key, (o, lse) in gqa.items():
        o_ref, lse_ref = mla_o[key]
        assert _max_abs(o, o_ref) < 1e-10 and abs(lse - lse_ref) < 1e-10
        u, _ = ua[key]
        assert _max_abs(W_UV_g[key[2] // hpg] @ u, o) < 1e-10
