"""Pins for the oracle's INT8 outlier side path ("LLM inference cost: W8A8/W4A8 ...",
sec. 2.2, second technique): the largest-magnitude 2% of each group's weights kept in
INT8 beside the INT4 tile and added back on a side path.

The page prints no worked example; the pins are a brute-force selection (numpy's stable
sort on (-|w|, k)), the INT8 closed forms, the dense remainder's invariants, a
reconstruction that is exact on constructed grids, the reduction to the plain INT4 path
with no outliers, and the side-path product against numpy's matmul of the dequantized
matrix.  They run on the CPU only.
"""
import numpy as np

import oracle


def _w(K, N, seed, outliers=True):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    if outliers:
        m = rng.random((K, N)) < 0.01
        W[m] *= 8.0
    return W


def test_count_is_two_percent_rounded_up():
    assert [oracle.outlier_count(g) for g in (128, 64, 256, 50, 100, 8)] == [3, 2, 6, 1, 2, 1]


def test_selection_matches_a_stable_sort():
    K, N, g = 256, 12, 128
    W = _w(K, N, 1)
    W[5, 0] = W[9, 0] = 2.0           # a tie for the largest |w|: the smaller k ranks first
    W[130, 1], W[200, 1] = -3.0, 3.0  # a tie of opposite signs
    idx, c8, s8, dense, st = oracle.outlier_split(W, group=g)
    assert st == 0
    c = oracle.outlier_count(g)
    for gi in range(K // g):
        blk = W[gi * g:(gi + 1) * g]
        for n in range(N):
            order = np.lexsort((np.arange(g), -np.abs(blk[:, n])))  # by -|w|, then k
            np.testing.assert_array_equal(idx[gi, :, n], order[:c])
    assert list(idx[0, :2, 0]) == [5, 9]
    assert list(idx[1, :2, 1]) == [130 - 128, 200 - 128]


def test_int8_codes_closed_form():
    K, N, g = 384, 20, 128
    W = _w(K, N, 2)
    idx, c8, s8, dense, st = oracle.outlier_split(W, group=g)
    assert st == 0
    G, c = K // g, idx.shape[1]
    for gi in range(G):
        for n in range(N):
            vals = W[gi * g + idx[gi, :, n].astype(np.int64), n]
            want_s = np.float32(np.abs(vals).max()) / np.float32(127.0)
            assert s8[gi, n] == want_s
            assert abs(int(c8[gi, 0, n])) == 127            # the largest outlier takes the end code
            err = np.abs(vals.astype(np.float64) - c8[gi, :, n].astype(np.float64) * float(s8[gi, n]))
            assert np.all(err <= float(s8[gi, n]) / 2 * (1 + 2 ** -20))


def test_dense_remainder():
    K, N, g = 256, 10, 128
    W = _w(K, N, 3)
    idx, c8, s8, dense, st = oracle.outlier_split(W, group=g)
    assert st == 0
    for gi in range(K // g):
        for n in range(N):
            ks = gi * g + idx[gi, :, n].astype(np.int64)
            assert np.all(dense[ks, n] == 0.0)
            rest = np.setdiff1d(np.arange(gi * g, (gi + 1) * g), ks)
            np.testing.assert_array_equal(dense[rest, n], W[rest, n])
            assert np.abs(W[rest, n]).max() <= np.abs(W[ks, n]).min()


def test_no_outliers_is_the_plain_int4_path():
    K, N, M = 256, 16, 3
    W = _w(K, N, 4)
    X = np.random.default_rng(4).standard_normal((M, K)).astype(np.float32)
    idx, c8, s8, dense, st = oracle.outlier_split(W, count=0)
    assert st == 0
    np.testing.assert_array_equal(dense, W)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(dense)
    packed = oracle.pack_nibbles(codes)
    y, b = oracle.gemm_w4a16_outlier_ref(X, packed, scales, zeros, idx, c8, s8)
    y0, b0 = oracle.gemm_w4a16_ref(X, packed, scales, zeros)
    np.testing.assert_array_equal(y, y0)
    np.testing.assert_array_equal(b, b0)


def _dequant_full(codes, scales, zeros, idx, c8, s8, g=128):
    """Dense fp64 matrix deq4 + scatter(deq8), written with numpy."""
    K, N = codes.shape
    sc = oracle.f16_to_f32(scales).astype(np.float64)
    w = (codes.astype(np.float64) - np.repeat(zeros.astype(np.float64), g, axis=0)) * np.repeat(sc, g, axis=0)
    G, c, _ = idx.shape
    for gi in range(G):
        for r in range(c):
            k = gi * g + idx[gi, r].astype(np.int64)
            w[k, np.arange(N)] += c8[gi, r].astype(np.float64) * s8[gi].astype(np.float64)
    return w


def test_side_path_product_against_numpy():
    K, N, M = 384, 24, 5
    W = _w(K, N, 5)
    X = np.random.default_rng(5).standard_normal((M, K)).astype(np.float32)
    idx, c8, s8, dense, st = oracle.outlier_split(W)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(dense)
    y, b = oracle.gemm_w4a16_outlier_ref(X, oracle.pack_nibbles(codes), scales, zeros, idx, c8, s8)
    wd = _dequant_full(codes, scales, zeros, idx, c8, s8)
    np.testing.assert_allclose(y, X.astype(np.float64) @ wd, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(b, np.abs(X.astype(np.float64)) @ np.abs(wd), rtol=1e-12)


def test_exact_reconstruction_on_grids():
    """Every group: dense values on the INT4 grid of scale 1 spanning [-7, 8], and three
    outliers 254, -128 and 10, i.e. 127, -64 and 5 times s8 = 254 / 127 = 2.  Then
    deq4 + deq8 reproduces W exactly."""
    rng = np.random.default_rng(6)
    K, N, g = 256, 8, 128
    W = rng.integers(-7, 9, (K, N)).astype(np.float32)
    for gi in range(K // g):
        for n in range(N):
            lo, hi = rng.choice(np.arange(3, g), 2, replace=False)
            W[gi * g + lo, n], W[gi * g + hi, n] = -7.0, 8.0
            W[gi * g + 0, n], W[gi * g + 1, n], W[gi * g + 2, n] = 254.0, -128.0, 10.0
    idx, c8, s8, dense, st = oracle.outlier_split(W)
    assert st == 0
    assert np.all(s8 == 2.0)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(dense)
    np.testing.assert_array_equal(_dequant_full(codes, scales, zeros, idx, c8, s8), W.astype(np.float64))


def test_outliers_shrink_the_int4_range():
    """The point of the side path: with the outliers out, each group's INT4 scale is no
    larger, and on weights with 1% x8 outliers the total reconstruction error drops."""
    K, N = 512, 64
    W = _w(K, N, 7)
    codes0, scales0, zeros0, _ = oracle.quantize_w4_asym(W)
    idx, c8, s8, dense, st = oracle.outlier_split(W)
    codes1, scales1, zeros1, _ = oracle.quantize_w4_asym(dense)
    assert np.all(oracle.f16_to_f32(scales1) <= oracle.f16_to_f32(scales0))
    w0 = _dequant_full(codes0, scales0, zeros0, idx[:, :0], c8[:, :0], s8)
    w1 = _dequant_full(codes1, scales1, zeros1, idx, c8, s8)
    e0 = np.sum((w0 - W) ** 2)
    e1 = np.sum((w1 - W) ** 2)
    assert e1 < 0.5 * e0
