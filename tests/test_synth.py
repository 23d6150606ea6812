"""Host checks of the seeded input generator (no attention arithmetic here)."""
import numpy as np
import torch

from mla_latent_kv_23_b200 import synth


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 65504.0, 1e-30, 3.0e38], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(synth.bf16_round(x), want)
    assert np.array_equal(synth.from_bf16_bits(synth.bf16_bits(want)), want)


def test_permuted_block_table_uses_every_page_once():
    w = synth.config("ragged").with_(B=9, len_range=(1, 700))
    L = synth.draw_seqlens(w)
    bt, n = synth.make_block_table(w, L)
    used = bt[bt >= 0]
    assert n == sum((int(l) + 63) // 64 for l in L)
    assert np.array_equal(np.sort(used), np.arange(n))
    assert np.all(L >= 1) and np.all(L <= 700)


def test_draws_are_reproducible_and_independent_of_other_sizes():
    w = synth.config("v3").with_(B=2, seqlens=(100, 70), d_model=64)
    a = synth.draw(w)
    b = synth.draw(w)
    assert np.array_equal(a["cache"], b["cache"]) and np.array_equal(a["W_Q"], b["W_Q"])
    c = synth.draw(w.with_(d_model=96))          # other tensor sizes change ...
    assert np.array_equal(a["cache"], c["cache"])  # ... the cache does not


def test_outlier_rows_scaled_by_eight():
    w = synth.config("long").with_(B=2, seqlens=(3000, 2000), d_model=8)
    x = synth.draw(w, with_weights=False)["cache"]
    base = synth.draw(w.with_(outlier_frac=0.0), with_weights=False)["cache"]
    ratio = np.abs(x).sum(1) / np.maximum(np.abs(base).sum(1), 1e-30)
    scaled = np.isclose(ratio, 8.0, rtol=1e-2)
    assert scaled.sum() == 50                     # 1% of the 5000 valid rows
    assert np.all(np.isclose(ratio[~scaled], 1.0))


def test_query_positions():
    w = synth.config("mtp").with_(B=3, seqlens=(10, 20, 30), d_model=8)
    d = synth.draw(w, with_weights=False)
    assert d["qpos"].tolist() == [[8, 9], [18, 19], [28, 29]]
