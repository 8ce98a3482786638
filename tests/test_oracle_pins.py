"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each test pins one oracle function to something other than itself: a hand-derived
worked example (tests/golden/hand_examples.json), a closed-form bound, brute force
over all codes on small inputs, a special case that reduces to a library matmul,
or an invariant of the SmoothQuant transform.  None of them re-types the oracle's
own formula.  They run on the CPU only.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        return json.load(f)


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# IEEE conversions (the fp16 scale storage and the bf16 output)
# ---------------------------------------------------------------------------
def _edge_floats():
    vals = [0.0, -0.0, 1.0, -1.0, 65504.0, 65505.0, 65519.99, 65520.0, 70000.0, -70000.0, 1e30, -1e30,
            2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 1e-30, -1e-30, 0.2, 1 / 3, -1 / 3,
            float("inf"), float("-inf")]
    rng = np.random.default_rng(7)
    rnd = (rng.standard_normal(4000) * np.exp(rng.uniform(-20, 12, 4000))).astype(np.float32)
    return np.concatenate([np.array(vals, np.float32), rnd])


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_f16_round_up_matches_ieee_definition():
    """RU(x) is the least binary16 >= x: numpy's round-to-nearest conversion, moved up one
    representable step (np.nextafter in float16) whenever it landed below x."""
    xs = _edge_floats()
    got = oracle.f32_to_f16_ru(xs)
    for x, g in zip(xs, got):
        h = np.float16(x)
        if np.isfinite(x) and float(h) < float(x):
            h = np.nextafter(h, np.float16(np.inf))
        want = np.array([h], np.float16).view(np.uint16)[0]
        assert g == want, (x, hex(g), hex(want))


def test_f16_decode_is_exact_on_every_pattern():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7C00) != 0x7C00
    dec = np.array([oracle.lib().qgo_f16_to_f32(int(b)) for b in bits[finite]], np.float32)
    np.testing.assert_array_equal(dec, bits[finite].view(np.float16).astype(np.float32))
    # and RU of an exact binary16 value is that value
    some = bits[finite][::97]
    back = oracle.f32_to_f16_ru(some.view(np.float16).astype(np.float32))
    ok = (back == some) | ((some == 0x8000) & (back == 0x8000))
    assert ok.all()


def test_bf16_round_to_nearest_even_matches_torch():
    xs = _edge_floats()
    # add exact ties between two bf16 neighbours
    base = np.array([1.0, 3.0, -5.0, 1e-3], np.float32).view(np.uint32)
    ties = (base + np.uint32(0x8000)).view(np.float32)
    ties_odd = (base + np.uint32(0x18000)).view(np.float32)
    xs = np.concatenate([xs, ties, ties_odd])
    got = oracle.f32_to_bf16_rn(xs)
    want = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# O1: asymmetric INT4 per group
# ---------------------------------------------------------------------------
def _column(group_vals, pad, K=128):
    col = np.full(K, pad, np.float32)
    col[: len(group_vals)] = group_vals
    return col.reshape(K, 1)


@pytest.mark.parametrize("case", range(2))
def test_w4_asym_hand_examples(case):
    ex = _hand()["w4_asym"][case]
    W = _column(ex["group"], ex["pad_value"])
    codes, scales, zeros, st = oracle.quantize_w4_asym(W)
    assert st == oracle.OK
    assert scales[0, 0] == int(ex["scale_f16_bits"], 16)
    assert zeros[0, 0] == ex["zero"]
    assert list(codes[: len(ex["codes"]), 0]) == ex["codes"]
    assert (codes[len(ex["codes"]):, 0] == ex["pad_code"]).all()


def _asym_weights(K=256, N=96, seed=3):
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=seed)
    # a few special groups: constant, all-zero, all-positive, all-negative, tiny range
    W[0:128, 0] = 0.37
    W[0:128, 1] = 0.0
    W[0:128, 2] = np.abs(W[0:128, 2]) + 0.5
    W[0:128, 3] = -np.abs(W[0:128, 3]) - 0.5
    if K >= 256:
        W[128:256, 4] = 1e-6 * np.arange(128, dtype=np.float32)
    return W


def test_w4_asym_round_trip_bound_and_ranges():
    """|x - (q - z) s| <= s/2 (1 + 2^-18) for every element (scale rounded up), z in [0, 15],
    and the fp16 scale covers the range: 15 s >= max' - min'."""
    W = _asym_weights()
    codes, scales, zeros, st = oracle.quantize_w4_asym(W)
    assert st == oracle.OK
    K, N = W.shape
    s = np.repeat(_f16(scales), 128, axis=0)
    z = np.repeat(zeros.astype(np.float64), 128, axis=0)
    xhat = (codes.astype(np.float64) - z) * s
    err = np.abs(W.astype(np.float64) - xhat)
    assert (err <= s / 2 * (1 + 2.0 ** -18) + 0.0).all()
    assert (zeros <= 15).all() and (codes <= 15).all()
    Wg = W.astype(np.float64).reshape(K // 128, 128, N)
    r = np.maximum(Wg.max(axis=1), 0) - np.minimum(Wg.min(axis=1), 0)
    assert (15 * _f16(scales) >= r * (1 - 2.0 ** -22)).all()
    # a constant group has one exact code for its value; a zero group has scale 0
    assert xhat[0, 0] == pytest.approx(0.37, abs=_f16(scales)[0, 0] / 2)
    assert scales[0, 1] == 0 and (codes[0:128, 1] == 0).all()


def test_w4_asym_brute_force_nearest_grid_point():
    """Each code is the nearest of the 16 grid points (j - z) s; only near-ties (within the
    binary32 rounding of x/s) may pick the other neighbour."""
    W = _asym_weights(K=128, N=64, seed=11)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(W)
    s = _f16(scales)[0]
    z = zeros[0].astype(np.float64)
    x = W.astype(np.float64)
    grid = (np.arange(16)[:, None, None] - z[None, None, :]) * s[None, None, :]  # [16,1,N]
    d = np.abs(x[None] - grid)  # [16,K,N]
    best = d.argmin(axis=0)
    dq = np.take_along_axis(d, codes[None].astype(np.int64), 0)[0]
    dbest = d.min(axis=0)
    near_tie = (dq - dbest) <= s[None, :] * 2.0 ** -19
    live = s[None, :] > 0
    assert ((codes == best) | near_tie | ~live).all()


def test_w4_asym_grid_points_are_fixed_points():
    """dequantize -> quantize is the identity on grid points of a scale that fp16 holds exactly."""
    rng = np.random.default_rng(5)
    N = 32
    s = (2.0 ** rng.integers(-8, 0, N)).astype(np.float32) * np.float32(1.5)   # exact in fp16
    z = rng.integers(0, 16, N)
    q = rng.integers(0, 16, (128, N))
    q[0, :] = 0
    q[1, :] = 15          # span the full range so that s = (max - min)/15 exactly
    W = ((q - z[None, :]) * s[None, :]).astype(np.float32)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(W)
    # reading A: the range includes 0, which the grid does since z in [0, 15]
    np.testing.assert_array_equal(_f16(scales)[0], s.astype(np.float64))
    np.testing.assert_array_equal(zeros[0], z)
    np.testing.assert_array_equal(codes, q)


def test_w4_asym_monotone_and_nonfinite():
    x = np.linspace(-1.0, 2.0, 128, dtype=np.float32).reshape(128, 1)
    codes, _, _, _ = oracle.quantize_w4_asym(x)
    assert (np.diff(codes[:, 0].astype(int)) >= 0).all()
    bad = _asym_weights(K=128, N=8)
    bad[5, 3] = np.nan
    assert oracle.quantize_w4_asym(bad)[3] == oracle.NONFINITE
    big = np.full((128, 1), 1e6, np.float32)
    big[0, 0] = -1e6
    assert oracle.quantize_w4_asym(big)[3] == oracle.RANGE


def test_w4_smoothed_input_equals_prescaled_input():
    """Quantizing diag(s) W with s passed in equals quantizing the pre-multiplied matrix."""
    W = _asym_weights(K=256, N=40)
    s = np.random.default_rng(2).uniform(0.2, 5.0, 256).astype(np.float32)
    a = oracle.quantize_w4_asym(W, s_smooth=s)
    b = oracle.quantize_w4_asym(W * s[:, None])
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


# ---------------------------------------------------------------------------
# O1s: symmetric INT4
# ---------------------------------------------------------------------------
def test_w4_sym_hand_example():
    ex = _hand()["w4_sym"][0]
    W = _column(ex["group"], ex["pad_value"])
    codes, scales, st = oracle.quantize_w4_sym(W)
    assert st == oracle.OK and scales[0, 0] == ex["scale"]
    assert list(codes[: len(ex["codes"]), 0]) == ex["codes"]


def test_w4_sym_absmax_bound_brute_force():
    W = synth.weights(256, 80, 0.02, 0.01, 8.0, seed=9)
    W[0:128, 7] = 0.0
    codes, scales, st = oracle.quantize_w4_sym(W)
    assert st == oracle.OK
    x = W.astype(np.float64)
    s = np.repeat(scales.astype(np.float64), 128, axis=0)
    assert (np.abs(codes) <= 7).all()
    assert (np.abs(x - codes * s) <= s / 2 * (1 + 2.0 ** -18)).all()
    # the largest |w| of each nonzero group codes to +-7 with the sign of w
    g = x.reshape(2, 128, 80)
    am = np.abs(g).argmax(axis=1)
    c = codes.reshape(2, 128, 80)
    for gi in range(2):
        for n in range(80):
            if scales[gi, n] > 0:
                assert c[gi, am[gi, n], n] == 7 * np.sign(g[gi, am[gi, n], n])
    assert scales[0, 7] == 0 and (codes[0:128, 7] == 0).all()
    # brute force: nearest of the 15 grid points j*s, j in [-7, 7]
    grid = np.arange(-7, 8)[:, None, None] * s[None]
    d = np.abs(x[None] - grid)
    dq = np.take_along_axis(d, (codes.astype(np.int64) + 7)[None], 0)[0]
    assert ((dq - d.min(axis=0)) <= s * 2.0 ** -19).all()


# ---------------------------------------------------------------------------
# O2: packing
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", range(2))
def test_pack_hand_words(case):
    ex = _hand()["pack"][case]
    codes = np.array(ex["codes_k0_to_k7"], np.int64).astype(np.int8).view(np.uint8).reshape(8, 1)
    assert int(oracle.pack_nibbles(codes)[0, 0]) == int(ex["word"], 16)


def test_pack_unpack_bijection():
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, (256, 24)).astype(np.uint8)
    p = oracle.pack_nibbles(codes)
    assert p.shape == (32, 24)
    np.testing.assert_array_equal(oracle.unpack_nibbles(p, 256), codes)
    # column n of word row kb only depends on codes[8kb:8kb+8, n]
    codes2 = codes.copy()
    codes2[9, 5] ^= 0xF
    p2 = oracle.pack_nibbles(codes2)
    diff = np.argwhere(p2 != p)
    assert diff.tolist() == [[1, 5]] and (p2[1, 5] ^ p[1, 5]) == 0xF << 4


# ---------------------------------------------------------------------------
# O3: W4A16 GEMM reference
# ---------------------------------------------------------------------------
def test_w4a16_ref_reduces_to_integer_matmul():
    """Power-of-two scales, z = 8 and small integer X make every product and partial sum
    exact: the reference must equal numpy's int64 matmul, scaled, bit for bit."""
    rng = np.random.default_rng(4)
    M, K, N = 3, 256, 40
    q = rng.integers(0, 16, (K, N)).astype(np.uint8)
    e = rng.integers(-6, 3, (K // 128, N))
    scales = np.array(2.0 ** e, np.float16).view(np.uint16)
    zeros = np.full((K // 128, N), 8, np.uint8)
    X = rng.integers(-8, 9, (M, K))
    packed = oracle.pack_nibbles(q)
    y, b = oracle.gemm_w4a16_ref(X.astype(np.float32), packed, scales, zeros)
    wint = q.astype(np.int64) - 8
    scale_full = np.repeat(2.0 ** e, 128, axis=0)
    # exact: split K by group, integer matmul per group, times the per-(g, n) power of two
    want = np.zeros((M, N))
    want_b = np.zeros((M, N))
    for g in range(K // 128):
        sl = slice(128 * g, 128 * (g + 1))
        want += (X[:, sl] @ wint[sl]) * 2.0 ** e[g]
        want_b += (np.abs(X[:, sl]) @ np.abs(wint[sl])) * 2.0 ** e[g]
    np.testing.assert_array_equal(y, want)
    np.testing.assert_array_equal(b, want_b)
    # and the row subset path selects rows, not columns
    y2, _ = oracle.gemm_w4a16_ref(X.astype(np.float32), packed, scales, zeros, rows=[2, 0])
    np.testing.assert_array_equal(y2, want[[2, 0]])
    assert scale_full.shape == (K, N)


def test_w4a16_ref_matches_library_matmul_of_dequantized_weights():
    W = synth.weights(256, 48, 0.02, 0.01, 8.0, seed=21)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(W)
    packed = oracle.pack_nibbles(codes)
    X, _ = synth.activations(5, 256, "bf16", seed=21)
    s = np.repeat(_f16(scales), 128, axis=0)
    z = np.repeat(zeros.astype(np.float64), 128, axis=0)
    wd = (codes.astype(np.float64) - z) * s
    y, b = oracle.gemm_w4a16_ref(X, packed, scales, zeros)
    np.testing.assert_allclose(y, X.astype(np.float64) @ wd, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b, np.abs(X.astype(np.float64)) @ np.abs(wd), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# O4: SmoothQuant factors
# ---------------------------------------------------------------------------
def _smooth_case():
    cfg = synth.CONFIGS["w8a8"]
    K, N = 256, 96
    Xcal, _ = synth.activations(64, K, "bf16", channels=8, mult=50.0, seed=3)
    W = synth.weights(K, N, 0.02, seed=3)
    return Xcal, W, cfg


def test_smooth_half_alpha_equalises_ranges():
    """At alpha = 0.5, max_m |X~_j| = max_n |W~_j| = sqrt(max|X_j| max|W_j|) (to 2 ulp):
    the transform moves the difficulty from activations to weights exactly half way."""
    Xcal, W, _ = _smooth_case()
    s, inv, st = oracle.smooth_scales(Xcal, W, 0.5)
    assert st == oracle.OK
    ax = np.abs(Xcal.astype(np.float64)).max(axis=0)
    aw = np.abs(W.astype(np.float64)).max(axis=1)
    lhs = ax * inv.astype(np.float64)
    rhs = aw * s.astype(np.float64)
    geo = np.sqrt(ax * aw)
    np.testing.assert_allclose(lhs, geo, rtol=4 * 2.0 ** -24)
    np.testing.assert_allclose(rhs, geo, rtol=4 * 2.0 ** -24)


def test_smooth_identity_in_fp64():
    """X W = (X diag(s)^-1)(diag(s) W) to 1e-12 relative in fp64 with the oracle's s, inv_s."""
    Xcal, W, _ = _smooth_case()
    s, inv, _ = oracle.smooth_scales(Xcal, W, 0.5)
    X, _ = synth.activations(16, 256, "bf16", channels=8, mult=50.0, seed=4)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    lhs = Xd @ Wd
    rhs = (Xd * (1.0 / s.astype(np.float64))) @ (Wd * s.astype(np.float64)[:, None])
    np.testing.assert_allclose(rhs, lhs, rtol=1e-12, atol=1e-12 * np.abs(lhs).max())
    # inv_s is 1/s to one rounding
    np.testing.assert_allclose(inv.astype(np.float64) * s.astype(np.float64), 1.0, rtol=2.0 ** -23)


def test_smooth_alpha_endpoints_and_zero_columns():
    Xcal, W, _ = _smooth_case()
    Xcal = Xcal.copy()
    Xcal[:, 5] = 0.0
    ax = np.abs(Xcal.astype(np.float64)).max(axis=0)
    aw = np.abs(W.astype(np.float64)).max(axis=1)
    s1, _, _ = oracle.smooth_scales(Xcal, W, 1.0)   # s_j = max|X_j|
    s0, _, _ = oracle.smooth_scales(Xcal, W, 0.0)   # s_j = 1 / max|W_j|
    live = ax > 0
    np.testing.assert_array_equal(s1[live], ax[live].astype(np.float32))
    np.testing.assert_allclose(s0[live], 1.0 / aw[live], rtol=2.0 ** -23)
    assert s1[5] == 1.0 and s0[5] == 1.0


# ---------------------------------------------------------------------------
# O5 / O6: symmetric INT8, per token and per output channel
# ---------------------------------------------------------------------------
def test_act_i8_hand_example():
    ex = _hand()["act_i8"][0]
    row = np.zeros((1, 128), np.float32)
    row[0, : len(ex["row"])] = ex["row"]
    q, t, st = oracle.smooth_quant_act_i8(row)
    assert st == oracle.OK and t[0] == ex["scale"]
    assert list(q[0, : len(ex["codes"])]) == ex["codes"] and (q[0, len(ex["codes"]):] == 0).all()


def test_act_i8_closed_form_and_brute_force():
    X, _ = synth.activations(12, 256, "bf16", channels=8, mult=50.0, seed=5)
    X[3] = 0.0
    inv = np.random.default_rng(0).uniform(0.05, 2.0, 256).astype(np.float32)
    q, t, st = oracle.smooth_quant_act_i8(X, inv)
    assert st == oracle.OK
    xt = X.astype(np.float64) * inv.astype(np.float64)            # exact product
    amax = np.abs(xt).max(axis=1)
    np.testing.assert_allclose(t.astype(np.float64) * 127, amax, rtol=2.0 ** -22)
    td = t.astype(np.float64)[:, None]
    assert (np.abs(q) <= 127).all()
    live = t > 0
    err = np.abs(xt - q * td)[live]
    assert (err <= td[live] / 2 * (1 + 2.0 ** -18) + 2.0 ** -24 * np.abs(xt[live])).all()
    am = np.abs(xt).argmax(axis=1)
    for m in np.nonzero(live)[0]:
        assert abs(int(q[m, am[m]])) == 127
    assert t[3] == 0 and (q[3] == 0).all()
    # without smoothing: same as smoothing by ones
    qa, ta, _ = oracle.smooth_quant_act_i8(X)
    qb, tb, _ = oracle.smooth_quant_act_i8(X, np.ones(256, np.float32))
    np.testing.assert_array_equal(qa, qb)
    np.testing.assert_array_equal(ta, tb)


def test_w8_channel_closed_form():
    W = synth.weights(256, 64, 0.02, seed=6)
    W[:, 9] = 0.0
    s = np.random.default_rng(1).uniform(0.3, 3.0, 256).astype(np.float32)
    Wq, sw, st = oracle.quantize_w8_channel(W, s)
    assert st == oracle.OK
    wt = W.astype(np.float64) * s.astype(np.float64)[:, None]
    np.testing.assert_allclose(sw.astype(np.float64) * 127, np.abs(wt).max(axis=0), rtol=2.0 ** -22)
    live = sw > 0
    err = np.abs(wt - Wq * sw.astype(np.float64)[None, :])[:, live]
    assert (err <= sw[live] / 2 * (1 + 2.0 ** -18) + 2.0 ** -24 * np.abs(wt[:, live])).all()
    am = np.abs(wt).argmax(axis=0)
    assert all(abs(int(Wq[am[n], n])) == 127 for n in np.nonzero(live)[0])
    assert sw[9] == 0 and (Wq[:, 9] == 0).all()


# ---------------------------------------------------------------------------
# O7 / O8: integer GEMMs
# ---------------------------------------------------------------------------
def test_w8a8_accumulator_and_reference():
    rng = np.random.default_rng(8)
    M, K, N = 5, 384, 72
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    Wq = rng.integers(-127, 128, (K, N)).astype(np.int8)
    t = rng.uniform(0.01, 1.0, M).astype(np.float32)
    sw = rng.uniform(0.001, 0.01, N).astype(np.float32)
    acc, y, yref, b = oracle.gemm_w8a8(Xq, t, Wq, sw)
    exact = Xq.astype(np.int64) @ Wq.astype(np.int64)
    np.testing.assert_array_equal(acc, exact)
    xd = Xq.astype(np.float64) * t.astype(np.float64)[:, None]
    wd = Wq.astype(np.float64) * sw.astype(np.float64)[None, :]
    np.testing.assert_allclose(yref, xd @ wd, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b, np.abs(xd) @ np.abs(wd), rtol=1e-12)
    yv = y.view(np.uint16).astype(np.uint32) << 16
    assert oracle.within_tolerance(yv.view(np.float32), yref, b).all()
    # unit scales: the output is the accumulator rounded once to bf16 (torch's conversion)
    _, y1, _, _ = oracle.gemm_w8a8(Xq, np.ones(M, np.float32), Wq, np.ones(N, np.float32))
    want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(y1, want)


def test_w4a8_partials_and_reference():
    rng = np.random.default_rng(10)
    M, K, N = 4, 384, 40
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    q = rng.integers(-7, 8, (K, N)).astype(np.int8)
    sg = rng.uniform(0.001, 0.01, (K // 128, N)).astype(np.float32)
    t = rng.uniform(0.01, 1.0, M).astype(np.float32)
    packed = oracle.pack_nibbles(q)
    part, yref, b = oracle.gemm_w4a8(Xq, t, packed, sg)
    for g in range(K // 128):
        sl = slice(128 * g, 128 * (g + 1))
        np.testing.assert_array_equal(part[:, g, :], Xq[:, sl].astype(np.int64) @ q[sl].astype(np.int64))
    xd = Xq.astype(np.float64) * t.astype(np.float64)[:, None]
    wd = q.astype(np.float64) * np.repeat(sg.astype(np.float64), 128, axis=0)
    np.testing.assert_allclose(yref, xd @ wd, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(b, np.abs(xd) @ np.abs(wd), rtol=1e-12)


def _bf16_bits_of_f64(v):
    # f64 -> f32 is exact for the values used here; then torch's RNE conversion to bf16
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_w4a8_output_exact_case_is_rounded_integer_product():
    """Power-of-two group and token scales with small integer codes make every binary32
    product and partial sum of the W4A8 output exact, so the output must be the exact
    product (numpy's int64 matmul per group, scaled) rounded once to bf16."""
    rng = np.random.default_rng(12)
    M, K, N = 5, 8192, 24
    Xq = rng.integers(-31, 32, (M, K)).astype(np.int8)
    q = rng.integers(-7, 8, (K, N)).astype(np.int8)
    e = rng.integers(-2, 1, (K // 128, N))
    sg = (2.0 ** e).astype(np.float32)
    t = (2.0 ** rng.integers(-9, -5, M)).astype(np.float32)
    packed = oracle.pack_nibbles(q)
    _, yref, _, y = oracle.gemm_w4a8(Xq, t, packed, sg, want_part=False, want_y=True)
    exact = np.zeros((M, N))
    for g in range(K // 128):
        sl = slice(128 * g, 128 * (g + 1))
        exact += (Xq[:, sl].astype(np.int64) @ q[sl].astype(np.int64)) * 2.0 ** e[g]
    exact *= t.astype(np.float64)[:, None]
    np.testing.assert_array_equal(yref, exact)
    np.testing.assert_array_equal(y, _bf16_bits_of_f64(exact))


def test_w4a8_output_sums_groups_in_ascending_order_in_binary32():
    """Hand example: three groups whose scaled partials are 2^24, 1 and -2^24.  In
    binary32 and ascending group order, 2^24 + 1 rounds to 2^24 (tie to even) and the
    output is exactly 0; any other order, or a binary64 sum, gives 1."""
    K, N = 384, 1
    Xq = np.zeros((1, K), np.int8)
    q = np.zeros((K, N), np.int8)
    Xq[0, 0:128] = 64
    q[0:128, 0] = 2             # P0 = 128 * 64 * 2 = 16384
    Xq[0, 128] = 1
    q[128, 0] = 1               # P1 = 1
    Xq[0, 256:384] = 64
    q[256:384, 0] = -2          # P2 = -16384
    sg = np.array([[1024.0], [1.0], [1024.0]], np.float32)
    t = np.ones(1, np.float32)
    part, yref, _, y = oracle.gemm_w4a8(Xq, t, oracle.pack_nibbles(q), sg, want_y=True)
    np.testing.assert_array_equal(part[0, :, 0], [16384, 1, -16384])
    assert yref[0, 0] == 1.0
    assert int(y[0, 0]) == 0x0000


def test_w4a8_output_within_tolerance_of_reference():
    rng = np.random.default_rng(13)
    M, K, N = 6, 1024, 64
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    q = rng.integers(-7, 8, (K, N)).astype(np.int8)
    sg = rng.uniform(0.001, 0.01, (K // 128, N)).astype(np.float32)
    t = rng.uniform(0.01, 1.0, M).astype(np.float32)
    _, yref, b, y = oracle.gemm_w4a8(Xq, t, oracle.pack_nibbles(q), sg, want_part=False, want_y=True)
    yv = (y.astype(np.uint32) << 16).view(np.float32)
    assert oracle.within_tolerance(yv, yref, b).all()
    # one bf16 rounding of a binary32 sum: within 2^-8 relative of the fp64 value, plus the
    # binary32 summation error, far inside the tolerance
    assert (np.abs(yv - yref) <= 2.0 ** -8 * np.abs(yref) + 1e-4 * b).all()


def test_f64_gemm_matches_numpy():
    X, _ = synth.activations(3, 128, "bf16", seed=1)
    W = synth.weights(128, 20, 0.02, seed=1)
    np.testing.assert_allclose(oracle.gemm_f64(X, W), X.astype(np.float64) @ W.astype(np.float64), rtol=1e-12,
                               atol=1e-14)
