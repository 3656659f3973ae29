"""The seeded input recipe: determinism, distributions, and low-rank quality."""

import numpy as np

import synth


def test_streams_are_deterministic_and_distinct():
    a = synth.normal(3, 1, 1000)
    b = synth.normal(3, 1, 1000)
    c = synth.normal(3, 2, 1000)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert np.array_equal(synth.normal(3, 1, 10), a[:10])
    # chunked generation equals one-shot generation
    assert np.array_equal(synth.normal(3, 1, 1000, chunk=64), a)


def test_normal_moments():
    z = synth.normal(0, 9, 1 << 20)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    u = synth.uniform(0, 9, 1 << 20)
    assert 0 <= u.min() and u.max() < 1 and abs(u.mean() - 0.5) < 2e-3


def test_outlier_structure():
    d = synth.svdq_layer(0, 256, 1024, 64, 8, x_out_frac=0.01, x_out_scale=20.0,
                         w_out_rows=8, w_out_scale=10.0)
    assert len(d["x_outliers"]) == 10
    x = synth.bf16_bits_to_f32(d["x"])
    col = np.abs(x).max(axis=0)
    assert set(np.argsort(col)[-10:]) == set(d["x_outliers"].tolist())
    lam = d["lam"]
    # smoothing moves the outlier channels' magnitude into the weights
    assert lam[d["x_outliers"]].min() > np.median(lam)


def test_low_rank_factors_near_eckart_young():
    """L1 L2 from the randomized SVD is close to the best rank-r approximation
    of diag(lambda) W (Eckart-Young: its error is the tail singular values)."""
    d = synth.svdq_layer(1, 64, 256, 192, 16, w_out_rows=4, w_out_scale=10.0)
    What = d["lam"].astype(np.float64)[:, None] * d["W"].astype(np.float64)
    s = np.linalg.svd(What, compute_uv=False)
    best = np.sqrt((s[16:] ** 2).sum())
    L1 = synth.bf16_bits_to_f32(d["L1"]).astype(np.float64)
    L2 = synth.bf16_bits_to_f32(d["L2"]).astype(np.float64)
    err = np.linalg.norm(What - L1 @ L2)
    assert best <= err <= best * 1.01


def test_qkv_epilogue_inputs():
    a = synth.qkv_epilogue_inputs(2, 64, 128, 24)
    b = synth.qkv_epilogue_inputs(2, 64, 128, 24)
    assert np.array_equal(a["wq"], b["wq"]) and not np.array_equal(a["wq"], a["wk"])
    w = synth.bf16_bits_to_f32(a["wq"])
    assert w.shape == (128,) and (w >= 0.5).all() and (w <= 1.5).all()
    assert a["cos"].shape == (64, 64) and a["sin"].dtype == np.float32
    # position 0 is not rotated; every (cos, sin) pair is a unit vector
    assert (a["cos"][0] == 1).all() and (a["sin"][0] == 0).all()
    assert np.allclose(a["cos"].astype(np.float64) ** 2 + a["sin"].astype(np.float64) ** 2, 1, atol=1e-6)
