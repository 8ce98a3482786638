"""GPU parity of the AWQ scale search ("Quantization & Flash Attention -- LLM inference
optimization (2)", sec. 2.1-2.3) against the CPU oracle, through the C ABI.

Bit-exact: the per-channel statistic (a binary64 sum in token order on both sides, one
rounding), the scaled activations (one fp32 product, one bf16 rounding), and the scales
at alpha = 0 and 1.  Other exponents: within 1 ulp (binary64 pow from two libraries,
rounded once to fp32).

The MSE per grid point: the device's quantized output is bf16 (the W4A16 GEMM's output
dtype) and its reference X W accumulates in fp32, while the oracle keeps both in
binary64.  The bf16 rounding e of an output y is at most half an ulp (|e| <= 2^-9 |y|);
with e uncorrelated with the quantization error D, it adds E[e^2] ~ (2^-8 |y|)^2 / 12 to
E[D^2], i.e. ~1e-3 of the MSE at |y| / rms(D) ~ 30.  The tests allow a relative 2e-2.
The winner: several grid points are correct when their MSEs lie within that tolerance
of the least one; the device's pick must be one of them, must be the oracle's pick when
no other point is that close, and the returned scales must be the oracle's scales at
the device's pick.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import cuda, x_device

pytestmark = pytest.mark.gpu

MSE_RTOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_quantized_gemm_group_b200 as q
    assert q.qg_device_status() == q.QG_OK


def qlib():
    import bit_quantized_gemm_group_b200 as q
    return q


def _status_ok():
    q = qlib()
    st = q.qg_device_status()
    assert st == q.QG_OK, q.qg_status_string(st)


def _ulps(a, b):
    """Distance in units in the last place between two arrays of positive fp32."""
    return np.abs(np.asarray(a, np.float32).view(np.int32).astype(np.int64) -
                  np.asarray(b, np.float32).view(np.int32).astype(np.int64))


def _calib(K=4096, tokens=None):
    cfg = synth.CONFIGS["awq"]
    Xf, Xb = synth.calibration(K, cfg)
    if tokens is not None:
        Xf, Xb = Xf[:tokens].copy(), Xb[:tokens].copy()
    return Xf, Xb


def _rand_layer(Mc, K, N, seed):
    X, Xb = synth.activations(Mc, K, "bf16", channels=max(1, K // 256), mult=40.0, seed=seed)
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=seed)
    return X, Xb, W


def _search(Xb, W, n_grid):
    q = qlib()
    Mc, K = Xb.shape
    mse = torch.full((n_grid,), float("nan"), dtype=torch.float64, device="cuda")
    best = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    s = torch.full((K,), float("nan"), dtype=torch.float32, device="cuda")
    inv = torch.full((K,), float("nan"), dtype=torch.float32, device="cuda")
    q.qg_awq_search(x_device(Xb, torch.bfloat16), cuda(W), n_grid, mse, best, s, inv)
    _status_ok()
    return mse.cpu().numpy(), int(best.item()), s.cpu().numpy(), inv.cpu().numpy()


def _check_search(Xf, Xb, W, n_grid):
    mse, b, s, inv = _search(Xb, W, n_grid)
    mse_o, best_o, _, _, st = oracle.awq_search(Xf, W, n_grid)
    assert st == 0
    np.testing.assert_allclose(mse, mse_o, rtol=MSE_RTOL)
    near = [i for i in range(n_grid) if mse_o[i] <= mse_o.min() * (1 + 2 * MSE_RTOL)]
    assert b in near, (b, near, mse_o)
    if len(near) == 1:
        assert b == best_o
    s_at, inv_at = oracle.awq_scales(oracle.awq_act_mean(Xf), oracle.awq_alpha(b, n_grid))
    assert _ulps(s, s_at).max() <= 1
    assert _ulps(inv, inv_at).max() <= 2
    return mse, b


def test_act_mean_bitexact_on_the_calibration_batch():
    q = qlib()
    for Xf, Xb in [_calib(), synth.activations(3, 100, "bf16", channels=2, mult=50.0, seed=9)]:
        Mc, K = Xf.shape
        xm = torch.full((K,), float("nan"), dtype=torch.float32, device="cuda")
        q.qg_awq_act_mean(x_device(Xb, torch.bfloat16), xm)
        _status_ok()
        np.testing.assert_array_equal(xm.cpu().numpy(), oracle.awq_act_mean(Xf))


@pytest.mark.parametrize("alpha", [0.0, 1.0, 0.5, 0.35, 0.05, 0.95])
def test_scales(alpha):
    q = qlib()
    Xf, _ = _calib()
    xm = oracle.awq_act_mean(Xf)
    xm[[3, 17]] = 0.0  # zero statistics keep s = 1
    s = torch.empty(xm.size, dtype=torch.float32, device="cuda")
    inv = torch.empty_like(s)
    q.qg_awq_scales(cuda(xm), alpha, s, inv)
    _status_ok()
    s_o, inv_o = oracle.awq_scales(xm, alpha)
    if alpha in (0.0, 1.0):
        np.testing.assert_array_equal(s.cpu().numpy(), s_o)
        np.testing.assert_array_equal(inv.cpu().numpy(), inv_o)
    else:
        assert _ulps(s.cpu().numpy(), s_o).max() <= 1
        assert _ulps(inv.cpu().numpy(), inv_o).max() <= 2
    assert s.cpu().numpy()[3] == 1.0 and s.cpu().numpy()[17] == 1.0


def test_scale_act_bitexact():
    q = qlib()
    Xf, Xb = _calib()
    _, inv = oracle.awq_scales(oracle.awq_act_mean(Xf), 0.5)
    Xs = torch.empty(Xf.shape, dtype=torch.bfloat16, device="cuda")
    q.qg_awq_scale_act(x_device(Xb, torch.bfloat16), cuda(inv), Xs)
    _status_ok()
    got = Xs.cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, oracle.awq_scale_act(Xf, inv))


@pytest.mark.parametrize("Mc,K,N,n_grid", [(64, 256, 64, 11), (40, 384, 136, 6), (160, 256, 136, 4),
                                            (1, 128, 8, 1), (7, 128, 24, 2)])
def test_search_small(Mc, K, N, n_grid):
    """Ragged column counts, one-group K, a single token, a one-point grid, and a
    calibration batch large enough for the tile GEMM (160 tokens)."""
    Xf, Xb, W = _rand_layer(Mc, K, N, seed=Mc + K + N)
    _check_search(Xf, Xb, W, n_grid)


def test_search_finds_the_exact_layer():
    """alpha = 1 makes the constructed layer exact: scaled weights on the INT4 grid and
    scaled activations +-1, so only the bf16 output rounding remains there."""
    rng = np.random.default_rng(0)
    Mc, K, N = 8, 128, 16
    e = rng.integers(-2, 4, K)
    X = (np.where(rng.random((Mc, K)) < 0.5, -1.0, 1.0) * np.exp2(e)[None, :]).astype(np.float32)
    qv = rng.integers(-7, 9, (K, N))
    for n in range(N):
        lo, hi = rng.choice(K, 2, replace=False)
        qv[lo, n], qv[hi, n] = -7, 8
    W = (qv * np.exp2(-e)[:, None]).astype(np.float32)
    Xb = (X.view(np.uint32) >> 16).astype(np.uint16)  # powers of two: exact in bf16
    mse, b, s, _ = _search(Xb, W, 5)
    assert b == 4
    assert mse[4] <= 0.05 * mse[:4].min()
    np.testing.assert_array_equal(s, np.exp2(e).astype(np.float32))


def test_search_on_the_workload_shape_sampled_tokens():
    """The decode layer's full weight (4096 x 12288) against the first 32 calibration
    tokens, three grid points (the oracle's binary64 GEMMs bound the size)."""
    cfg = synth.CONFIGS["awq"]
    K, N = cfg["KN"][0]
    Xf, Xb = _calib(K, tokens=32)
    W = synth.workload_weights("awq", K, N)
    mse, b = _check_search(Xf, Xb, W, 3)
    assert mse[b] < mse[0]  # the method's claim on outlier channels: some alpha > 0 beats plain INT4


def test_search_is_repeatable():
    Xf, Xb, W = _rand_layer(48, 256, 72, seed=3)
    a = _search(Xb, W, 7)
    b = _search(Xb, W, 7)
    np.testing.assert_array_equal(a[0], b[0])
    assert a[1] == b[1]
    np.testing.assert_array_equal(a[2], b[2])
