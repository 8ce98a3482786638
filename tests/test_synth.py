"""The seeded input recipe (CPU): the generators draw what each workload describes --
weight spread and outlier fraction, activation outlier channels, the storage rounding
of X -- deterministically per (seed, role, shape), and the exact-arithmetic operands
stay inside the bounds that make every GEMM product and partial sum exact."""
import numpy as np
import pytest
import torch

import synth


@pytest.mark.parametrize("name", ["w4a16_tiny", "w4a16_decode", "w4a16_prefill", "w8a8", "w4a8", "awq"])
def test_weight_spread_and_outliers(name):
    cfg = synth.CONFIGS[name]
    K, N = 1024, 2048
    W = synth.workload_weights(name, K, N, seed=3)
    assert W.dtype == np.float32 and W.shape == (K, N)
    frac, mult = cfg.get("outlier_frac", 0.0), cfg.get("outlier_mult", 1.0)
    # W is the N(0, std) draw with the entries of an independent Bernoulli(frac) mask
    # scaled by mult: rebuilt here from the two role streams
    mask = synth.rng(3, synth.S_MASK, K, N).random((K, N), dtype=np.float32) < np.float32(frac)
    base = synth.rng(3, synth.S_W, K, N).standard_normal((K, N), dtype=np.float32) * np.float32(cfg["w_std"])
    want = base.copy()
    want[mask] *= np.float32(mult)
    np.testing.assert_array_equal(W, want)
    n = K * N
    assert abs(mask.sum() - frac * n) <= 5 * np.sqrt(max(frac * (1 - frac) * n, 1.0))  # binomial, 5 sigma
    assert abs(float(base.std()) - cfg["w_std"]) < 0.01 * cfg["w_std"]


@pytest.mark.parametrize("name", ["w8a8", "w4a8", "w4a16_decode"])
def test_activation_channels_and_rounding(name):
    cfg = synth.CONFIGS[name]
    M, K = 64, 4096
    vals, bits = synth.workload_activations(name, M, K, seed=5)
    assert vals.shape == (M, K) and bits.dtype == np.uint16
    # the stored values are the 16-bit patterns, read back exactly
    dt = torch.bfloat16 if cfg["xdtype"] == "bf16" else torch.float16
    back = torch.from_numpy(bits.view(np.int16)).view(dt).to(torch.float32).numpy()
    np.testing.assert_array_equal(back, vals)
    ch = synth.outlier_channels(K, cfg.get("x_channels", 0), seed=5)
    assert len(ch) == cfg.get("x_channels", 0) and len(set(ch.tolist())) == len(ch)
    if len(ch):
        rest = np.setdiff1d(np.arange(K), ch)
        ratio = np.abs(vals[:, ch]).mean() / np.abs(vals[:, rest]).mean()
        assert abs(ratio - cfg["x_mult"]) < 0.15 * cfg["x_mult"]
        # the calibration batch shares the channels but not the draws
        cal, _ = synth.calibration(K, cfg, seed=5)
        assert cal.shape == (cfg["calib_tokens"], K)
        assert np.abs(cal[:, ch]).mean() / np.abs(cal[:, rest]).mean() > 0.8 * cfg["x_mult"]
        assert not np.array_equal(cal[:M], vals)


def test_draws_are_deterministic_and_role_separated():
    a = synth.weights(256, 128, 0.02, 0.01, 8.0, seed=7)
    b = synth.weights(256, 128, 0.02, 0.01, 8.0, seed=7)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, synth.weights(256, 128, 0.02, 0.01, 8.0, seed=8))
    x1, _ = synth.activations(4, 256, seed=7)
    x2, _ = synth.activations(4, 256, seed=7, stream=synth.S_XCAL)
    assert not np.array_equal(x1, x2)


def test_exact_operands_stay_in_bounds():
    K, N = 512, 256
    codes, scales, zeros = synth.exact_w4_asym(K, N, seed=1)
    assert codes.min() >= 0 and codes.max() <= 15 and zeros.max() <= 15
    s = scales.view(np.float16).astype(np.float64)
    assert set(np.unique(np.log2(s)).tolist()) <= {-2.0, -1.0, 0.0}
    c8, s8 = synth.exact_w4_sym(K, N, seed=1)
    assert c8.min() >= -7 and c8.max() <= 7 and set(np.unique(np.log2(s8)).tolist()) <= {-2.0, -1.0, 0.0}
    X, bits = synth.exact_activations(16, K, seed=1)
    assert np.abs(X).max() <= 8 and np.array_equal(X, np.round(X))
    np.testing.assert_array_equal(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy(), X)
    Xq, t = synth.exact_act_i8(16, K, seed=1)
    assert np.abs(Xq.astype(np.int32)).max() <= 31
    assert set(np.unique(np.log2(t)).tolist()) <= {-9.0, -8.0, -7.0, -6.0}
