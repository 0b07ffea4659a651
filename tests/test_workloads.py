"""Host checks of the seeded input generator: the static quantization recipes it applies.

The per-tensor percentile recipe (x clipped at a percentile of |x|, B and C by their absmax,
one scale each) is the Quamba per-tensor baseline on Mamba-2 that the Quamba2 OpenReview
rebuttal describes alongside its Table R9; the per-head recipe is the SSDi8 page's per-H(G) axis.
"""
import numpy as np
import pytest

from quantized_mamba_ssd_b200 import workloads as W


def test_percentile_scale_is_the_percentile_over_all_tokens_when_few():
    rng = np.random.default_rng(1)
    v = rng.laplace(size=(2, 300, 4, 8)).astype(np.float32)
    s = W.percentile_scale(v, 99.9)
    assert s == np.float32(np.percentile(np.abs(v), 99.9) / 127.0)


def test_percentile_scale_calibrates_on_evenly_spaced_tokens():
    rng = np.random.default_rng(2)
    L = 3 * W.CALIB_TOKENS + 5
    v = rng.normal(size=(1, L, 2, 4)).astype(np.float32)
    s = W.percentile_scale(v, 99.0)
    step = -(-L // W.CALIB_TOKENS)
    assert s == np.float32(np.percentile(np.abs(v[:, ::step]), 99.0) / 127.0)


def test_percentile_workload_saturates_the_tail_and_uses_one_scale():
    c = W.make_prefill(2, 2000, 8, 64, 32, 2, 256, law="laplace_outliers_all",
                       scales="percentile", clip_percentile=99.99, seed=4)
    # one scale per tensor, broadcast over heads and groups
    for s in (c.x_scale, c.B_scale, c.C_scale):
        assert (s == s[0]).all() and s[0] > 0
    # about 1e-4 of x lands on +-127 (the clipped tail plus the values that round to the end)
    sat = (np.abs(c.x.astype(np.int32)) == 127).mean()
    assert 0.8e-4 <= sat <= 3e-4, sat
    assert np.abs(c.x.astype(np.int32)).max() == 127 and c.x.min() >= -127
    # B and C by absmax: the largest value maps to exactly +-127 and nothing is clipped
    for q in (c.B, c.C):
        assert np.abs(q.astype(np.int32)).max() == 127
        assert (np.abs(q.astype(np.int32)) == 127).mean() < 1e-3


def test_clipping_enlarges_x_codes_and_leaves_B_C_alone():
    # the same activations under the absmax and the clipped per-tensor recipes
    c = W.make_prefill(1, 200, 4, 64, 16, 1, 64, law="laplace_outliers_x", scales="percentile",
                       clip_percentile=99.0, seed=5)
    ref = W.make_prefill(1, 200, 4, 64, 16, 1, 64, law="laplace_outliers_x", scales="tensor",
                         seed=5)
    # a smaller scale: no code of the clipped recipe is smaller in magnitude
    assert (np.abs(c.x.astype(np.int32)) >= np.abs(ref.x.astype(np.int32))).all()
    assert c.x_scale[0] < ref.x_scale[0]
    assert np.array_equal(c.B, ref.B) and np.array_equal(c.C, ref.C)


def test_generation_is_seeded():
    a = W.make_prefill(1, 100, 4, 64, 16, 2, 64, law="laplace_outliers_all",
                       scales="percentile", seed=9)
    b = W.make_prefill(1, 100, 4, 64, 16, 2, 64, law="laplace_outliers_all",
                       scales="percentile", seed=9)
    for f in ("x", "B", "C", "dt", "A", "D", "x_scale", "B_scale", "C_scale"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_unknown_scale_recipe_is_rejected():
    with pytest.raises(ValueError):
        W.make_prefill(1, 8, 2, 64, 16, 1, 64, scales="per-channel")


def test_varlen_lengths_fill_the_tokens_within_bounds():
    for seed in range(5):
        n = W.varlen_lengths(32768, 64, 8192, seed)
        assert n.sum() == 32768 and n.max() <= 8192 and n.min() >= 1
        assert (n[:-1] >= 64).all()  # only the last one is cut
    assert W.varlen_lengths(0, 64, 8192, 0).size == 0


def test_varlen_config_is_seeded_and_packed():
    case, cu = W.make_varlen_config(total_tokens=3000)
    case2, cu2 = W.make_varlen_config(total_tokens=3000)
    assert np.array_equal(cu, cu2) and np.array_equal(case.x, case2.x)
    assert cu[0] == 0 and cu[-1] == 3000 and (np.diff(cu) > 0).all()
    assert case.batch == 1 and case.seqlen == 3000 and case.x.dtype == np.int8


def test_channel_scales_quantize_each_dstate_channel():
    c = W.make_prefill(2, 50, 4, 8, 6, 2, 64, law="laplace_outliers_all", scales="channel", seed=3)
    assert c.B_scale.shape == (2, 6) and c.C_scale.shape == (2, 6) and c.x_scale.shape == (4,)
    # every (group, channel) slice reaches the full code range, so its scale is its own absmax
    for q in (c.B, c.C):
        assert (np.abs(q.astype(np.int16)).max(axis=(0, 1)) == 127).all()
    # the per-head path keeps its scales and codes bit for bit
    a = W.make_prefill(2, 50, 4, 8, 6, 2, 64, law="laplace_outliers_all", scales="head", seed=3)
    assert np.array_equal(a.x, c.x) and np.array_equal(a.x_scale, c.x_scale)
    assert a.B_scale.shape == (2,)


def test_oracle_runs_on_channel_scales():
    import oracle
    c = W.make_prefill(1, 40, 4, 3, 6, 2, 64, law="normal", scales="channel", seed=4)
    y, fs, _ = oracle.scan(c.x, c.B, c.C, c.dt, c.A, c.D, c.x_scale, c.B_scale, c.C_scale)
    assert np.isfinite(y).all() and fs.shape == (1, 4, 3, 6)
