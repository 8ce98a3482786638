"""Pins for the oracle's GPTQ ("Quantization & Flash Attention -- LLM inference
optimization (2)", sec. 3.1-3.3): rows of W rounded one after another to the INT4 group
grid, each rounding error spread over the rows not yet rounded through the inverse
Hessian H = (2/n) X^T X + lambda I.

The page prints no worked example.  The pins:
* the Hessian on a hand-computed case;
* inputs with orthogonal channels (X^T X exactly diagonal): no compensation, so GPTQ
  equals plain round-to-nearest INT4 bit for bit;
* weights already on the INT4 grid: a fixed point;
* the Cholesky form of sec. 3.3 (numpy: upper factor of H^-1, row ratios U[k][j]/U[k][k])
  reaching the same codes, scales and zeros as the oracle's explicit eliminations;
* output columns rounded independently;
* the method's claim: a lower layer error ||X (W - W_hat)||^2 than round-to-nearest;
* the teacher-forced replay (the checker for results made elsewhere, e.g. on a GPU)
  accepts the oracle's own result and flags a code moved by one step or a scale moved by
  more than the allowed ulps.
They run on the CPU only.
"""
import numpy as np

import oracle


def _deq(codes, scales, zeros, g):
    sc = oracle.f16_to_f32(scales).astype(np.float64)
    return (codes.astype(np.float64) - np.repeat(zeros.astype(np.float64), g, axis=0)) * np.repeat(sc, g, axis=0)


def _correlated(M, K, seed):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((K, K)) * 0.3 + np.eye(K)
    return (rng.standard_normal((M, K)) @ A).astype(np.float32)


def test_hessian_hand_case():
    X = np.array([[1.0, 0.0, 2.0], [0.0, 3.0, 1.0], [1.0, 1.0, 0.0], [2.0, 0.0, 1.0]], np.float32)
    xtx = np.array([[6.0, 1.0, 4.0], [1.0, 10.0, 3.0], [4.0, 3.0, 6.0]])
    h = 2.0 / 4.0 * xtx
    lam = 0.01 * np.trace(h) / 3
    np.testing.assert_array_equal(oracle.gptq_hessian(X, 0.01), h + lam * np.eye(3))
    # all-zero inputs: the ridge alone
    np.testing.assert_array_equal(oracle.gptq_hessian(np.zeros((2, 3), np.float32), 0.01), 0.01 * np.eye(3))


def test_orthogonal_channels_reduce_to_round_to_nearest():
    K, N, g = 256, 24, 128
    rng = np.random.default_rng(1)
    c = rng.uniform(0.5, 4.0, K).astype(np.float32)
    X = np.zeros((2 * K, K), np.float32)
    X[np.arange(2 * K), np.arange(2 * K) % K] = np.tile(c, 2)  # one nonzero per row: X^T X diagonal
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    codes, scales, zeros, st = oracle.gptq(X, W, g)
    assert st == 0
    c0, s0, z0, _ = oracle.quantize_w4_asym(W, g)
    np.testing.assert_array_equal(codes, c0)
    np.testing.assert_array_equal(scales, s0)
    np.testing.assert_array_equal(zeros, z0)


def test_weights_on_the_grid_are_a_fixed_point():
    K, N, g = 256, 16, 128
    rng = np.random.default_rng(2)
    q = rng.integers(-7, 9, (K, N))
    for gi in range(K // g):
        for n in range(N):
            lo, hi = rng.choice(g, 2, replace=False)
            q[gi * g + lo, n], q[gi * g + hi, n] = -7, 8   # range [-7, 8]: scale 1, zero 7
    W = (q * 0.25).astype(np.float32)                        # scale 0.25 exactly
    codes, scales, zeros, st = oracle.gptq(_correlated(300, K, 2), W, g)
    assert st == 0
    np.testing.assert_array_equal(_deq(codes, scales, zeros, g), W.astype(np.float64))


def _gptq_cholesky(X, W, g, damp=0.01):
    """The Cholesky form (sec. 3.3) written with numpy: U upper with H^-1 = U^T U; row k
    rounded with the group's scale/zero (taken from the oracle's pinned quantizer on the
    group's compensated fp32 values), then W[j] -= (w_k - deq) * U[k][j] / U[k][k]."""
    K, N = W.shape
    H = oracle.gptq_hessian(X, damp)
    U = np.linalg.cholesky(np.linalg.inv(H)).T
    Wc = W.astype(np.float64).copy()
    codes = np.zeros((K, N), np.uint8)
    scales = np.zeros((K // g, N), np.uint16)
    zeros = np.zeros((K // g, N), np.uint8)
    for k in range(K):
        if k % g == 0:
            _, s16, z, _ = oracle.quantize_w4_asym(Wc[k:k + g].astype(np.float32), g)
            scales[k // g], zeros[k // g] = s16[0], z[0]
            s = oracle.f16_to_f32(s16[0]).astype(np.float32)
            zz = z[0].astype(np.int64)
        w = Wc[k].astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            qk = np.where(s != 0, np.clip(np.rint(w / s).astype(np.int64) + zz, 0, 15), 0)
        codes[k] = qk
        err = (Wc[k] - (qk - zz) * s.astype(np.float64)) / U[k, k]
        Wc[k + 1:] -= np.outer(U[k, k + 1:], err)
    return codes, scales, zeros


def test_cholesky_form_agrees():
    K, N, g = 256, 20, 128
    X = _correlated(400, K, 3)
    W = (np.random.default_rng(3).standard_normal((K, N)) * 0.02).astype(np.float32)
    codes, scales, zeros, st = oracle.gptq(X, W, g)
    assert st == 0
    c1, s1, z1 = _gptq_cholesky(X, W, g)
    np.testing.assert_array_equal(scales, s1)
    np.testing.assert_array_equal(zeros, z1)
    np.testing.assert_array_equal(codes, c1)


def test_columns_are_rounded_independently():
    K, N, g = 256, 12, 128
    X = _correlated(300, K, 4)
    W = (np.random.default_rng(4).standard_normal((K, N)) * 0.02).astype(np.float32)
    full = oracle.gptq(X, W, g)
    part = oracle.gptq(X, np.ascontiguousarray(W[:, 3:7]), g)
    for a, b in zip(full[:3], part[:3]):
        np.testing.assert_array_equal(a[:, 3:7], b)


def test_lower_layer_error_than_round_to_nearest():
    K, N, g = 256, 32, 128
    X = _correlated(512, K, 5)
    W = (np.random.default_rng(5).standard_normal((K, N)) * 0.02).astype(np.float32)
    codes, scales, zeros, st = oracle.gptq(X, W, g)
    c0, s0, z0, _ = oracle.quantize_w4_asym(W, g)
    Xd = X.astype(np.float64)
    e_gptq = np.sum((Xd @ (W - _deq(codes, scales, zeros, g))) ** 2)
    e_rtn = np.sum((Xd @ (W - _deq(c0, s0, z0, g))) ** 2)
    assert e_gptq < 0.7 * e_rtn


def test_replay_accepts_its_own_result_and_flags_a_changed_code():
    K, N, g = 256, 10, 128
    X = _correlated(300, K, 6)
    W = (np.random.default_rng(6).standard_normal((K, N)) * 0.02).astype(np.float32)
    codes, scales, zeros, st = oracle.gptq(X, W, g)
    assert oracle.gptq_replay(X, W, codes, scales, zeros, g, scale_ulps=0) == (0.0, 0, 0, 0)
    bad = codes.copy()
    k, n = 200, 3
    bad[k, n] = bad[k, n] + 1 if bad[k, n] < 15 else bad[k, n] - 1  # one step off: half a step outside
    slack, sm, zm, _ = oracle.gptq_replay(X, W, bad, scales, zeros, g, scale_ulps=0)
    assert slack >= 0.5 - 1e-9 and sm == 0 and zm == 0
    bad_s = scales.copy()
    bad_s[1, 4] += 3
    assert oracle.gptq_replay(X, W, codes, bad_s, zeros, g, scale_ulps=1)[1] >= 1
