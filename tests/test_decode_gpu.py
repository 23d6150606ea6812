"""GPU parity of the whole path (absorb -> query -> decode -> up-projection)
against the CPU oracle, at sizes the oracle finishes in seconds that still
span many 64-token tiles, ragged tails, several KV chunks and both query-row
counts, plus the edge cases of the method."""
import numpy as np
import pytest
import torch

from gpu_pipeline import (ATOL_REL, assert_parity, assert_tight, check_absorbed, check_expanded,
                          f64, lse_err, run_pipeline, to_dev, to_dev_i32)
from mla_latent_kv_23_b200 import mla, synth
from oracle import mla_oracle as orc

pytestmark = pytest.mark.gpu


def v3_small(**kw):
    base = dict(name="v3-small", B=3, s_q=1, n_h=128, d_model=512, d_c=512, d_h=128, d_v=128,
                d_R=64, page_size=64, dtype="bf16", seqlens=(100, 1000, 777),
                block_table="permuted", scale=1 / np.sqrt(192.0), seed=21)
    base.update(kw)
    return synth.Workload(**base)


def some_heads(w, heads_first=None, heads_rest=(0, 1, 63, 64, 127)):
    picks = []
    for b in range(w.B):
        hs = range(w.n_h) if (b == 0 and heads_first is None) else (heads_first if b == 0 else heads_rest)
        for r in range(w.s_q):
            for i in hs:
                if i < w.n_h:
                    picks.append((b, r, i))
    return picks


def test_tiny_config_full_pipeline():
    w = synth.config("tiny")
    inp = synth.draw(w)
    out = run_pipeline(w, inp)
    res = check_expanded(w, inp, out)
    assert res["n"] == w.B * w.n_h
    assert_parity(res)


@pytest.mark.parametrize("s_q", [1, 2])
@pytest.mark.parametrize("splits", [0, 1, 5])
def test_v3_shape_ragged(s_q, splits):
    w = v3_small(s_q=s_q)
    inp = synth.draw(w)
    out = run_pipeline(w, inp, num_splits=splits)
    p = mla.decode_params(out["q"], out["cache"], out["bt"], out["seqlens"], out["u"], out["lse"],
                          w.page_size, w.d_R, w.softmax_scale, splits)
    tc, _ = mla.mla_decode_kernel_info(p)
    assert tc == 1
    assert_parity(check_expanded(w, inp, out, some_heads(w)))


@pytest.mark.parametrize("s_q,seqlens", [(1, (1, 64, 65, 128, 129)), (2, (2, 64, 65, 130, 3))])
def test_length_edges(s_q, seqlens):
    # one token, exactly one tile, one tile + 1, two tiles, two tiles + 1;
    # checked on exact bf16 inputs (q from the generator) with the tight bound
    w = v3_small(s_q=s_q, B=len(seqlens), seqlens=seqlens, block_table="identity")
    inp = synth.draw(w)
    q = synth.random_q(w)
    out = run_pipeline(w, inp, q=to_dev(q, w))
    picks = [(b, r, i) for b in range(w.B) for r in range(s_q) for i in (0, 5, 64, 127)]
    assert_tight(check_absorbed(w, q, inp, out, picks, W_UV=inp["W_UV"]))


@pytest.mark.parametrize("s_q", [1, 2])
def test_length_edges_through_query_formation(s_q):
    w = v3_small(s_q=s_q, B=4, seqlens=(64, 65, 128, 129), block_table="identity")
    inp = synth.draw(w)
    out = run_pipeline(w, inp)
    assert_parity(check_expanded(w, inp, out, some_heads(w, heads_first=(0, 5, 127))))


def test_fewer_heads_and_bigger_pages():
    w = v3_small(n_h=16, page_size=256, seqlens=(300, 513, 256))
    inp = synth.draw(w)
    out = run_pipeline(w, inp)
    assert_parity(check_expanded(w, inp, out))


def test_garbage_past_sequence_end_is_ignored():
    w = v3_small(seqlens=(70, 200, 129), tail_fill="nan")
    inp = synth.draw(w)
    out = run_pipeline(w, inp)
    assert torch.isfinite(out["u"].float()).all() and torch.isfinite(out["lse"]).all()
    assert_parity(check_expanded(w, inp, out, some_heads(w, heads_first=(0, 77))))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("s_q,splits", [(1, 4), (1, 0), (2, 3)])
def test_small_latent_tensor_core_path(dtype, s_q, splits):
    # d_c = 64, d_R = 16 runs on the small-latent tcgen05 kernel: tf32 for
    # fp32 tensors, bf16 otherwise; a permuted block table, pages of 192
    # tokens, a ragged tail (129 = 2 tiles + 1) and split rows
    w = synth.config("tiny").with_(dtype=dtype, B=3, s_q=s_q, seqlens=(129, 129, 129),
                                   page_size=192, block_table="permuted", full_pipeline=False)
    inp = synth.draw(w)
    out = run_pipeline(w, inp, num_splits=splits)
    p = mla.decode_params(out["q"], out["cache"], out["bt"], out["seqlens"], out["u"], out["lse"],
                          w.page_size, w.d_R, w.softmax_scale, splits)
    tc, _ = mla.mla_decode_kernel_info(p)
    assert tc == 1
    res = check_expanded(w, inp, out)
    assert res["n"] == w.B * w.s_q * w.n_h
    assert_parity(res)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_small_latent_on_exact_inputs(dtype):
    # the same q on both sides, many tiles and chunks, s_q = 2 with lengths
    # that leave a query row's last tile empty (65 = 64 + 1)
    w = synth.Workload(name="small-exact", B=4, s_q=2, n_h=8, d_model=64, d_c=64, d_h=32,
                       d_v=32, d_R=16, page_size=64, dtype=dtype, seqlens=(65, 700, 2, 1000),
                       block_table="permuted", seed=9)
    inp = synth.draw(w)
    q = synth.random_q(w)
    out = run_pipeline(w, inp, num_splits=7, q=to_dev(q, w))
    picks = [(b, r, i) for b in range(w.B) for r in range(w.s_q) for i in range(w.n_h)]
    res = check_absorbed(w, q, inp, out, picks, W_UV=inp["W_UV"])
    if dtype == "bf16":
        assert_tight(res)
        return
    # fp32 tensors run as tf32 (10 stored significand bits): every product of
    # a score carries up to 2^-10 of each operand, so an lse (a smooth maximum
    # of scale * scores) can move by up to scale * 2^-9 * max_j sum_k |q_k c_jk|,
    # more than 1e-3 of an lse near 0; lse is held to the larger of the two
    assert res["o"] <= ATOL_REL and res["u"] <= ATOL_REL, res
    lse = f64(out["lse"])
    ref = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w, picks)
    for (b, r, i), (_, lse_ref) in ref.items():
        L = int(inp["seqlens"][b])
        rows = orc.gather_rows(inp["cache"], inp["block_table"], w.page_size, b, L - w.s_q + r + 1)
        tf32 = w.softmax_scale * 2.0 ** -9 * float(np.max(np.abs(rows) @ np.abs(q[b, r, i])))
        allow = max(1e-3 * max(abs(lse_ref), 1.0), tf32)
        assert abs(lse[b, r, i] - lse_ref) <= allow, (b, r, i, lse[b, r, i], lse_ref, allow)


def test_unsupported_latent_widths_are_refused():
    # no attend kernel for these shapes: refused before anything runs
    q = torch.zeros((1, 1, 8, 96 + 16), dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((64, 96 + 16), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    sl = torch.ones((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(mla.MLAError) as e:
        mla.decode(q, cache, bt, sl, 64, 16, 0.1)
    assert e.value.status == 2   # MLA_ERR_UNSUPPORTED


@pytest.mark.parametrize("u_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("s_q,splits", [(1, 0), (1, 7), (2, 0), (2, 3)])
def test_decode_on_exact_inputs_tight(s_q, splits, u_dtype):
    # same bf16 q on both sides: only the kernel's own rounding remains; u in
    # fp32 (fp32 split partials) or in bf16 (bf16 split partials)
    w = v3_small(s_q=s_q, B=5, seqlens=(100, 1000, 777, 64, 2))
    inp = synth.draw(w)
    q = synth.random_q(w)
    out = run_pipeline(w, inp, num_splits=splits, q=to_dev(q, w), u_dtype=u_dtype)
    assert out["u"].dtype == u_dtype
    picks = [(b, r, i) for b in range(w.B) for r in range(s_q) for i in (0, 1, 64, 127)]
    assert_tight(check_absorbed(w, q, inp, out, picks, W_UV=inp["W_UV"]))


@pytest.mark.parametrize("s_q,splits", [(1, 0), (1, 4), (2, 0)])
def test_running_max_jumps_across_tiles(s_q, splits):
    # The kernel keeps a stale running maximum and rescales O and the row sum
    # only when a tile's maximum exceeds it by a large factor.  Make every
    # head's score climb tile by tile: steps of about 2^20 (below that factor:
    # weights up to 2^20 accumulate unrescaled), 2^40 and 2^50 (above it: the
    # rescale must run), and drops (the maximum stays).  A skipped or wrong
    # rescale leaves earlier tiles weighted 2^30+ times too high.
    w = v3_small(s_q=s_q, B=3, seqlens=(1000, 777, 130))
    inp = synth.draw(w)
    q = synth.random_q(w)
    q[..., 0] = 16.0
    cache = inp["cache"].copy()
    rng = np.random.default_rng(5)
    for b, L in enumerate(inp["seqlens"]):
        n_t = (int(L) + 63) // 64
        gamma = np.cumsum(rng.choice([-12.0, 12.0, 24.0, 30.0], size=n_t))
        gamma -= gamma.min()
        rows = synth.cache_row_ids(w, inp["block_table"], b, int(L))
        cache[rows, 0] = gamma[np.arange(int(L)) // 64]
    inp["cache"] = synth.bf16_round(cache)
    out = run_pipeline(w, inp, num_splits=splits, q=to_dev(q, w))
    picks = [(b, r, i) for b in range(w.B) for r in range(s_q) for i in (0, 1, 64, 127)]
    assert_tight(check_absorbed(w, q, inp, out, picks, W_UV=inp["W_UV"]))


@pytest.mark.parametrize("T,d_v", [(1, 128), (16, 128), (33, 128), (100, 128), (17, 40), (16, 100), (3, 12)])
def test_up_projection_of_fp32_u(T, d_v):
    # an fp32 u (spread up to ~|u| 25 like the stress workload) against the
    # exact product: the two bf16 terms of u leave 2^-16 |u|, so only o's own
    # bf16 rounding (2^-8 |o|) and fp32 accumulation remain.  d_v below 128
    # (a multiple of 8: o leaves as 16-byte stores; else one value per store)
    w = v3_small(B=T, seqlens=(1,) * T, block_table="identity", d_v=d_v)
    inp = synth.draw(w)
    u = (np.random.default_rng(T).standard_normal((T, w.n_h, w.d_c)) * 8).astype(np.float32)
    W_UV = to_dev(inp["W_UV"], w)
    o = torch.empty((T, w.n_h, w.d_v), dtype=torch.bfloat16, device="cuda")
    mla.mla_up_proj(torch.from_numpy(u).cuda(), W_UV, o)
    mla.mla_check_device_errors()
    o_ref = orc.up_project(u, inp["W_UV"])
    absWu = np.einsum("thc,hvc->thv", np.abs(u).astype(np.float64), np.abs(inp["W_UV"]).astype(np.float64))
    err = np.abs(f64(o) - o_ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -14 * absWu + 1e-5)
    assert np.max(err / (1 + np.abs(o_ref))) <= ATOL_REL


@pytest.mark.parametrize("T", [1, 16, 64, 100])
def test_up_projection_on_exact_input(T):
    # the up-projection checked on its own bf16 input u (from the generator)
    w = v3_small(B=T, seqlens=(1,) * T, block_table="identity")
    inp = synth.draw(w)
    u = synth.random_q(w)[:, 0, :, :w.d_c] * 8   # spread up to ~|u| 25 like the stress workload
    u = synth.bf16_round(np.ascontiguousarray(u))
    W_UV = to_dev(inp["W_UV"], w)
    o = torch.empty((T, w.n_h, w.d_v), dtype=torch.bfloat16, device="cuda")
    mla.mla_up_proj(to_dev(u, w), W_UV, o)
    o_ref = orc.up_project(u, inp["W_UV"])
    err = np.abs(f64(o) - o_ref) / (1 + np.abs(o_ref))
    assert err.max() <= ATOL_REL
    # fp32 accumulation + bf16 output: within 2^-8 relative of |o| + fp32 terms
    assert np.all(np.abs(f64(o) - o_ref) <= 2.0 ** -8 * np.abs(o_ref) + 1e-3)


def test_split_count_and_page_permutation_invariance():
    w = v3_small(seqlens=(1500, 900, 2048), block_table="identity")
    inp = synth.draw(w)
    q = synth.random_q(w)
    qd = to_dev(q, w)
    cache = to_dev(inp["cache"], w)
    bt = to_dev_i32(inp["block_table"])
    sl = to_dev_i32(inp["seqlens"])
    outs = {}
    for splits in (1, 3, 16, 100):
        outs[splits] = mla.decode(qd, cache, bt, sl, w.page_size, w.d_R, w.softmax_scale, splits)
    u1, l1 = (f64(t) for t in outs[1])
    for s, (u, l) in outs.items():
        assert np.max(np.abs(f64(u) - u1) / (1 + np.abs(u1))) < ATOL_REL
        assert np.max(np.abs(f64(l) - l1) / np.abs(l1)) < 1e-4
    # same result bit for bit when the pages are moved and the table follows them
    perm = np.random.default_rng(3).permutation(inp["num_pages"])
    P = w.page_size
    cache2 = np.empty_like(inp["cache"])
    for p_old in range(inp["num_pages"]):
        cache2[perm[p_old] * P:(perm[p_old] + 1) * P] = inp["cache"][p_old * P:(p_old + 1) * P]
    bt2 = np.where(inp["block_table"] >= 0, perm[np.maximum(inp["block_table"], 0)], -1)
    u2, l2 = mla.decode(qd, to_dev(cache2, w), to_dev_i32(bt2), sl, w.page_size, w.d_R,
                        w.softmax_scale, 3)
    assert torch.equal(u2, outs[3][0]) and torch.equal(l2, outs[3][1])
    # and the decode matches the oracle's absorbed helper on the same query
    ref = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w,
                              [(b, 0, i) for b in range(w.B) for i in (0, 31, 127)])
    for (b, r, i), (u_ref, lse_ref) in ref.items():  # noqa: B007
        assert np.max(np.abs(u1[b, r, i] - u_ref) / (1 + np.abs(u_ref))) < ATOL_REL
        assert lse_err(l1[b, r, i], lse_ref) <= 1.0


def test_row0_of_two_query_rows_equals_shorter_single_row():
    w = v3_small(s_q=2, seqlens=(300, 64, 1025), block_table="identity")
    inp = synth.draw(w)
    q = to_dev(synth.random_q(w), w)
    cache, bt = to_dev(inp["cache"], w), to_dev_i32(inp["block_table"])
    u2, l2 = mla.decode(q, cache, bt, to_dev_i32(inp["seqlens"]), w.page_size, w.d_R,
                        w.softmax_scale, 1)
    u1, l1 = mla.decode(q[:, :1].contiguous(), cache, bt, to_dev_i32(inp["seqlens"] - 1),
                        w.page_size, w.d_R, w.softmax_scale, 1)
    assert torch.equal(u1[:, 0], u2[:, 0]) and torch.equal(l1[:, 0], l2[:, 0])


def test_device_flags_for_bad_inputs():
    w = v3_small(B=2, seqlens=(100, 200), block_table="identity")
    inp = synth.draw(w)
    q = to_dev(synth.random_q(w), w)
    cache = to_dev(inp["cache"], w)
    bt = inp["block_table"].copy()
    bt[1, 1] = inp["num_pages"] + 5          # page id out of range
    u, l = mla.decode(q, cache, to_dev_i32(bt), to_dev_i32(inp["seqlens"]), w.page_size, w.d_R,
                      w.softmax_scale)
    with pytest.raises(mla.MLAError) as e:
        mla.mla_check_device_errors()
    assert e.value.flags & mla.DEVFLAG_BAD_PAGE
    sl = inp["seqlens"].copy()
    sl[0] = 10 ** 6                          # longer than the block table allows
    u, l = mla.decode(q, cache, to_dev_i32(inp["block_table"]), to_dev_i32(sl), w.page_size,
                      w.d_R, w.softmax_scale)
    with pytest.raises(mla.MLAError) as e:
        mla.mla_check_device_errors()
    assert e.value.flags & mla.DEVFLAG_BAD_SEQLEN
    assert torch.all(u[0] == 0) and torch.all(torch.isneginf(l[0]))
    assert mla.mla_check_device_errors() == 0   # flags were cleared


def test_fp16_partials_out_of_range_are_flagged():
    # with an fp32 u the partial u of a split row is stored in fp16; latent
    # values beyond its range (here 1e5) raise MLA_DEVFLAG_RANGE, and a
    # batch within range raises nothing
    w = v3_small(B=1, seqlens=(700,), block_table="identity")
    inp = synth.draw(w)
    q = to_dev(synth.random_q(w), w)
    bt, sl = to_dev_i32(inp["block_table"]), to_dev_i32(inp["seqlens"])
    cache = to_dev(inp["cache"], w)
    mla.decode(q, cache, bt, sl, w.page_size, w.d_R, w.softmax_scale, 4)
    assert mla.mla_check_device_errors() == 0
    big = cache.clone()
    big[:, :w.d_c] *= 1e5
    mla.decode(q, big, bt, sl, w.page_size, w.d_R, w.softmax_scale, 4)
    with pytest.raises(mla.MLAError) as e:
        mla.mla_check_device_errors()
    assert e.value.flags & mla.DEVFLAG_RANGE
    # one chunk: the row is written whole in fp32, nothing to flag
    u, _ = mla.decode(q, big, bt, sl, w.page_size, w.d_R, w.softmax_scale, 1)
    assert mla.mla_check_device_errors() == 0
    assert torch.isfinite(u).all()


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    # the wait every kernel uses on its mbarriers: on a phase that completes
    # it returns at once; on one that never completes it gives up after its
    # limit, raises the timeout flag and the kernel ends; the next decode
    # runs and agrees with one taken before
    w = v3_small(B=2, seqlens=(100, 200), block_table="identity")
    inp = synth.draw(w)
    q = to_dev(synth.random_q(w), w)
    cache, bt, sl = to_dev(inp["cache"], w), to_dev_i32(inp["block_table"]), to_dev_i32(inp["seqlens"])
    u0, l0 = mla.decode(q, cache, bt, sl, w.page_size, w.d_R, w.softmax_scale)
    assert mla.mla_check_device_errors() == 0
    mla.mla_selftest_wait(True)
    assert mla.mla_check_device_errors() == 0
    mla.mla_selftest_wait(False)
    with pytest.raises(mla.MLAError) as e:
        mla.mla_check_device_errors()
    assert e.value.flags == mla.DEVFLAG_TIMEOUT
    assert mla.mla_check_device_errors() == 0   # flags were cleared
    u1, l1 = mla.decode(q, cache, bt, sl, w.page_size, w.d_R, w.softmax_scale)
    assert mla.mla_check_device_errors() == 0
    assert torch.equal(u0, u1) and torch.equal(l0, l1)


def test_empty_batch():
    q = torch.empty((0, 1, 128, 576), dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((64, 576), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((0, 1), dtype=torch.int32, device="cuda")
    sl = torch.zeros((0,), dtype=torch.int32, device="cuda")
    u, l = mla.decode(q, cache, bt, sl, 64, 64, 0.07)
    assert u.shape == (0, 1, 128, 512)


def test_absorb_and_query_against_oracle():
    w = v3_small(B=2, d_model=384, s_q=2, seqlens=(5000, 7))
    inp = synth.draw(w)
    from gpu_pipeline import absorb_and_query
    q, W_QK = absorb_and_query(w, inp)
    wqk_ref = orc.absorb_weights(inp["W_UK"], inp["W_Q"])
    e = np.abs(f64(W_QK) - wqk_ref) / (1e-2 + np.abs(wqk_ref))
    assert e.max() < 1e-2   # bf16 output rounding (2^-9) of an fp32-accumulated sum
    qd = f64(q)
    for b in range(w.B):
        for r in range(w.s_q):
            for i in (0, 100):
                qref = orc.absorbed_query(inp, w, b, r, i)
                assert np.max(np.abs(qd[b, r, i] - qref) / (1 + np.abs(qref))) < 2e-2


@pytest.mark.parametrize("world", [2, 3])
def test_context_pieces_decoded_apart_merge_to_the_whole(world):
    # context parallelism with its ranks emulated as separate decode calls on
    # one GPU: each call sees one contiguous page range of every sequence;
    # mla_merge_partials combines the partial (u, lse)
    from mla_latent_kv_23_b200 import shard
    w = v3_small(B=3, seqlens=(1000, 777, 4100))
    inp = synth.draw(w)
    q = synth.random_q(w)
    qd, cache = to_dev(q, w), to_dev(inp["cache"], w)
    us, ls = [], []
    for pieces in shard.split_context(inp["seqlens"], world, w.page_size):
        bt, sl = shard.local_tables(inp["block_table"], pieces, w.page_size)
        u_r, l_r = mla.decode(qd, cache, to_dev_i32(bt), to_dev_i32(sl), w.page_size, w.d_R,
                              w.softmax_scale)
        us.append(u_r)
        ls.append(l_r)
    u_parts, lse_parts = torch.stack(us).contiguous(), torch.stack(ls).contiguous()
    u, lse = torch.empty_like(us[0]), torch.empty_like(ls[0])
    mla.mla_merge_partials(u_parts, lse_parts, u, lse)
    mla.mla_check_device_errors()
    picks = [(b, 0, i) for b in range(w.B) for i in (0, 1, 64, 127)]
    ref = orc.decode_absorbed(q, inp["cache"], inp["block_table"], inp["seqlens"], w, picks)
    uu, ll = f64(u), f64(lse)
    for (b, r, i), (u_ref, lse_ref) in ref.items():
        assert np.max(np.abs(uu[b, r, i] - u_ref) / (1 + np.abs(u_ref))) <= ATOL_REL
        assert lse_err(ll[b, r, i], lse_ref) <= 1.0
    # and it agrees with one decode of the whole contexts
    u_full, l_full = mla.decode(qd, cache, to_dev_i32(inp["block_table"]),
                                to_dev_i32(inp["seqlens"]), w.page_size, w.d_R, w.softmax_scale)
    assert np.max(np.abs(uu - f64(u_full)) / (1 + np.abs(f64(u_full)))) <= ATOL_REL
    assert np.max(np.abs(ll - f64(l_full)) / np.maximum(np.abs(f64(l_full)), 1.0)) <= 1e-4


@pytest.mark.parametrize("dtype,d_c,R", [(torch.bfloat16, 512, 5), (torch.float32, 64, 3),
                                         (torch.bfloat16, 264, 40)])
def test_merge_partials_against_its_definition(dtype, d_c, R):
    # the merge on its own, against lse = log sum exp, u = sum exp(lse_r - lse) u_r in
    # fp64 on the same (rounded) inputs; parts marked -inf carry no weight and a
    # row whose parts are all -inf gives u = 0, lse = -inf
    g = torch.Generator().manual_seed(3)
    rows = 37
    u_parts = torch.randn((R, rows, d_c), generator=g).to(dtype)
    lse_parts = (torch.randn((R, rows), generator=g) * 20).float()
    lse_parts[0, 1] = -float("inf")
    lse_parts[:, 2] = -float("inf")
    u = torch.empty((rows, d_c), dtype=dtype, device="cuda")
    lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
    mla.mla_merge_partials(u_parts.cuda(), lse_parts.cuda(), u, lse)
    mla.mla_check_device_errors()
    up, lp = u_parts.double(), lse_parts.double()
    m = lp.max(dim=0).values
    ok = torch.isfinite(m)
    wts = torch.where(torch.isfinite(lp), torch.exp(lp - torch.where(ok, m, 0.0)), 0.0)
    z = wts.sum(dim=0)
    lse_ref = torch.where(ok, m + torch.log(torch.where(ok, z, 1.0)), -float("inf"))
    u_ref = torch.where(ok.unsqueeze(-1),
                        (wts.unsqueeze(-1) * up).sum(0) / torch.where(ok, z, 1.0).unsqueeze(-1), 0.0)
    got_u, got_l = u.double().cpu(), lse.double().cpu()
    assert torch.all(got_u[2] == 0) and got_l[2] == -float("inf")
    fin = ok.clone()
    assert torch.allclose(got_l[fin], lse_ref[fin], rtol=1e-6, atol=1e-5)
    # fp32 weights and sums, bf16 (2^-9) or fp32 output rounding
    tol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-5
    err = (got_u[fin] - u_ref[fin]).abs() / (1 + u_ref[fin].abs())
    assert err.max() <= tol


@pytest.mark.parametrize("s_q,splits,d_v", [(1, 0, 128), (1, 5, 128), (2, 0, 128), (2, 3, 128),
                                           (1, 5, 40), (2, 3, 100)])
def test_decode_step_fuses_the_combine_into_the_up_projection(s_q, splits, d_v):
    # mla_decode_step merges split rows inside the up-projection; it returns
    # what mla_decode followed by mla_up_proj returns, bit for bit (the same
    # arithmetic in the same order), and meets the oracle's bounds
    w = v3_small(s_q=s_q, B=5, seqlens=(100, 1000, 777, 64, 2), d_v=d_v)
    inp = synth.draw(w)
    q = synth.random_q(w)
    qd, cache = to_dev(q, w), to_dev(inp["cache"], w)
    bt, sl = to_dev_i32(inp["block_table"]), to_dev_i32(inp["seqlens"])
    W_UV = to_dev(inp["W_UV"], w)
    T = w.B * w.s_q
    u1, l1 = mla.decode(qd, cache, bt, sl, w.page_size, w.d_R, w.softmax_scale, splits)
    o1 = torch.empty((T, w.n_h, w.d_v), dtype=torch.bfloat16, device="cuda")
    mla.mla_up_proj(u1.view(T, w.n_h, w.d_c), W_UV, o1)
    u2, l2 = torch.full_like(u1, float("nan")), torch.full_like(l1, float("nan"))
    o2 = torch.full_like(o1, float("nan"))
    p = mla.decode_params(qd, cache, bt, sl, u2, l2, w.page_size, w.d_R, w.softmax_scale, splits)
    ws = torch.empty(mla.mla_decode_workspace_size(p), dtype=torch.uint8, device="cuda")
    mla.mla_decode_step(p, W_UV, o2, ws)
    mla.mla_check_device_errors()
    assert torch.equal(u1, u2) and torch.equal(l1, l2) and torch.equal(o1, o2)
    out = dict(u=u2, lse=l2, o=o2.view(w.B, w.s_q, w.n_h, w.d_v))
    picks = [(b, r, i) for b in range(w.B) for r in range(s_q) for i in (0, 1, 64, 127)]
    assert_tight(check_absorbed(w, q, inp, out, picks, W_UV=inp["W_UV"]))
