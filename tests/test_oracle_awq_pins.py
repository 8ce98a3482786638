"""Pins for the oracle's AWQ scale search ("Quantization & Flash Attention -- LLM
inference optimization (2)", sec. 2.1-2.3): s_c = mean|X_c|^alpha, alpha on a grid in
[0, 1], least output MSE of the INT4 layer.

The pages print no worked example, so the pins are closed forms and a constructed case
whose answer is known exactly:
* the statistic on inputs whose channel means are known in closed form;
* the scales at alpha = 0, 1, 1/2 on powers of two, and for zero channels;
* the grid's points;
* a layer where alpha = 1 makes every scaled weight an exact INT4 grid point and every
  scaled activation exact in bf16, so the quantized layer reproduces X W exactly: the
  MSE there is 0 and the search must pick alpha = 1;
* alpha = 0 reduces to the plain INT4 layer, composed here from the pinned quantizer
  and W4A16 reference;
* zero weights give equal MSEs everywhere, and the first grid point wins.
They run on the CPU only.
"""
import numpy as np

import oracle


def _bf16_exact(a):
    """Round an fp32 array to bf16 (the activations the layer sees) and back to fp32."""
    bits = oracle.f32_to_bf16_rn(np.asarray(a, np.float32))
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_act_mean_closed_form():
    M, K = 6, 20
    m = np.arange(M)[:, None]
    c = np.arange(K)[None, :]
    X = (np.where(m % 2 == 0, 1.0, -1.0) * (c + 1) * 0.25).astype(np.float32)
    X[:, 7] = 0.0
    X[:, 11] = np.where(np.arange(M) == 2, -3.0, 3.0)  # signs differ, magnitudes equal: mean 3
    xm = oracle.awq_act_mean(X)
    want = ((np.arange(K) + 1) * 0.25).astype(np.float32)
    want[7] = 0.0
    want[11] = 3.0
    np.testing.assert_array_equal(xm, want)
    # a mean over a non-power-of-two count rounds once from the exact value
    X3 = np.array([[1.0], [1.0], [-2.0]], np.float32)
    assert oracle.awq_act_mean(X3)[0] == np.float32(4.0 / 3.0)


def test_scales_closed_forms():
    xm = np.array([0.0, 1.0, 4.0, 0.25, 16.0, 3.0, 1e-20, 7.5], np.float32)
    s, inv = oracle.awq_scales(xm, 0.0)
    np.testing.assert_array_equal(s, np.ones_like(xm))
    np.testing.assert_array_equal(inv, np.ones_like(xm))
    s, inv = oracle.awq_scales(xm, 1.0)
    np.testing.assert_array_equal(s[1:], xm[1:])
    assert s[0] == 1.0  # a zero statistic keeps the channel unscaled
    np.testing.assert_array_equal(inv[1:], (np.float32(1.0) / xm[1:]).astype(np.float32))
    s, _ = oracle.awq_scales(np.array([4.0, 0.25, 16.0, 0.0], np.float32), 0.5)
    np.testing.assert_array_equal(s, np.array([2.0, 0.5, 4.0, 1.0], np.float32))
    # monotone in the statistic for 0 < alpha, flat at alpha = 0
    xs = np.sort(np.random.default_rng(3).uniform(0.01, 50, 200)).astype(np.float32)
    for a in (0.25, 0.5, 0.75):
        s, _ = oracle.awq_scales(xs, a)
        assert np.all(np.diff(s) >= 0)


def test_grid_points():
    assert [oracle.awq_alpha(i, 21) for i in (0, 10, 20)] == [0.0, 0.5, 1.0]
    assert [oracle.awq_alpha(i, 5) for i in range(5)] == [0.0, 0.25, 0.5, 0.75, 1.0]
    assert oracle.awq_alpha(0, 1) == 0.0


def test_scale_act_rounds_once_to_bf16():
    import torch
    rng = np.random.default_rng(4)
    X = _bf16_exact(rng.standard_normal((5, 64)) * 3)
    inv = rng.uniform(0.01, 4.0, 64).astype(np.float32)
    inv[:8] = [0.5, 2.0, 0.25, 1.0, 4.0, 0.125, 1.0, 0.5]  # powers of two: exact scaling
    got = oracle.awq_scale_act(X, inv)
    prod = torch.from_numpy(X) * torch.from_numpy(inv)[None, :]  # one fp32 product (torch)
    want = prod.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)  # torch's RNE conversion
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal((got[:, :8].astype(np.uint32) << 16).view(np.float32), X[:, :8] * inv[:8])


def _exact_case(seed=0, M=8, K=256, N=16):
    """X[m][c] = +-2^e_c (so mean|X_c| = 2^e_c) and W[c][n] = q[c][n] 2^-e_c with every
    group of 128 rows of every column of q spanning exactly [-7, 8]."""
    rng = np.random.default_rng(seed)
    e = rng.integers(-2, 4, K)
    sign = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    X = (sign * np.exp2(e)[None, :]).astype(np.float32)
    q = rng.integers(-7, 9, (K, N))
    for g in range(K // 128):
        for n in range(N):
            lo, hi = rng.choice(128, 2, replace=False)
            q[128 * g + lo, n] = -7
            q[128 * g + hi, n] = 8
    W = (q * np.exp2(-e)[:, None]).astype(np.float32)
    return X, W, q, e


def test_alpha_one_is_exact_on_the_constructed_layer():
    X, W, q, e = _exact_case()
    mse, best, s, inv, st = oracle.awq_search(X, W, n_grid=5)
    assert st == 0
    assert mse[4] == 0.0  # alpha = 1: Q(s W) == q exactly and X / s == +-1 exactly
    assert best == 4
    assert np.all(mse[:4] > 0.0)
    np.testing.assert_array_equal(s, np.exp2(e).astype(np.float32))
    np.testing.assert_array_equal(inv, np.exp2(-e).astype(np.float32))


def test_alpha_zero_is_the_plain_int4_layer():
    rng = np.random.default_rng(5)
    M, K, N = 12, 256, 24
    X = _bf16_exact(rng.standard_normal((M, K)) * np.where(rng.random(K) < 0.05, 20.0, 1.0))
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    mse, best, _, _, st = oracle.awq_search(X, W, n_grid=3)
    assert st == 0
    codes, scales, zeros, _ = oracle.quantize_w4_asym(W)
    yq, _ = oracle.gemm_w4a16_ref(X, oracle.pack_nibbles(codes), scales, zeros)
    yref = X.astype(np.float64) @ W.astype(np.float64)
    np.testing.assert_allclose(mse[0], np.mean((yref - yq) ** 2), rtol=1e-12)
    assert mse[best] == mse.min()
    assert best == int(np.argmin(mse))


def test_zero_weights_tie_goes_to_the_first_point():
    rng = np.random.default_rng(6)
    X = _bf16_exact(rng.standard_normal((4, 128)))
    W = np.zeros((128, 8), np.float32)
    mse, best, s, _, st = oracle.awq_search(X, W, n_grid=4)
    assert st == 0
    np.testing.assert_array_equal(mse, np.zeros(4))
    assert best == 0
    np.testing.assert_array_equal(s, np.ones(128, np.float32))


def test_search_agrees_with_its_candidates():
    rng = np.random.default_rng(8)
    M, K, N = 10, 256, 16
    X = _bf16_exact(rng.standard_normal((M, K)) * np.where(rng.random(K) < 0.05, 30.0, 1.0))
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    mse, best, s_b, inv_b, st = oracle.awq_search(X, W, n_grid=6)
    assert st == 0 and np.all(mse >= 0)
    xm = oracle.awq_act_mean(X)
    yref = oracle.gemm_f64(X, W)
    for i in range(6):
        s, inv = oracle.awq_scales(xm, oracle.awq_alpha(i, 6))
        m_i, st_i = oracle.awq_candidate_mse(X, W, s, inv, yref=yref)
        assert st_i == 0 and m_i == mse[i]
    s, inv = oracle.awq_scales(xm, oracle.awq_alpha(best, 6))
    np.testing.assert_array_equal(s_b, s)
    np.testing.assert_array_equal(inv_b, inv)
