"""GPU parity of GPTQ ("Quantization & Flash Attention -- LLM inference optimization (2)",
sec. 3.1-3.3) against the CPU oracle, through the C ABI.

The device path takes the oracle's steps in the oracle's order with every binary64 /
binary32 operation rounded on its own, so the codes, fp16 scales and zeros must match bit
for bit.  The teacher-forced replay of the device's result through the oracle's
compensation is checked as well (every code the rounding of its replayed value), and the
result must feed the W4A16 GEMM like any INT4 weight.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_f32, cuda, u16, x_device

pytestmark = pytest.mark.gpu


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


def _calib(Mc, K, seed):
    """Correlated calibration activations in bf16 (fp32 values, bf16 bit patterns)."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((K, K)) * 0.3 + np.eye(K)
    X = torch.from_numpy((rng.standard_normal((Mc, K)) @ A).astype(np.float32)).to(torch.bfloat16)
    return X.to(torch.float32).numpy().copy(), X.view(torch.int16).numpy().view(np.uint16).copy()


def _gptq(Xb, W, group):
    q = qlib()
    K, N = W.shape
    codes = torch.full((K, N), 255, dtype=torch.uint8, device="cuda")
    scales = torch.zeros((K // group, N), dtype=torch.int16, device="cuda")
    zeros = torch.full((K // group, N), 255, dtype=torch.uint8, device="cuda")
    q.qg_gptq(x_device(Xb, torch.bfloat16), cuda(W), codes, scales, zeros, group=group)
    _status_ok()
    return codes, scales, zeros


@pytest.mark.parametrize("Mc,K,N,group", [(300, 256, 40, 128), (64, 128, 24, 64), (200, 256, 136, 32),
                                          (17, 384, 8, 128)])
def test_bitexact(Mc, K, N, group):
    X, Xb = _calib(Mc, K, seed=K + N)
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=N)
    codes, scales, zeros = _gptq(Xb, W, group)
    c_o, s_o, z_o, st = oracle.gptq(X, W, group)
    assert st == 0
    np.testing.assert_array_equal(codes.cpu().numpy(), c_o)
    np.testing.assert_array_equal(u16(scales), s_o)
    np.testing.assert_array_equal(zeros.cpu().numpy(), z_o)
    slack, sm, zm, st = oracle.gptq_replay(X, W, codes.cpu().numpy(), u16(scales), zeros.cpu().numpy(), group,
                                           scale_ulps=0)
    assert (slack, sm, zm, st) == (0.0, 0, 0, 0)


def test_feeds_the_w4a16_gemm_with_a_lower_layer_error():
    q = qlib()
    Mc, K, N, M = 256, 1024, 256, 16
    X, Xb = _calib(Mc, K, seed=5)
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=5)
    codes, scales, zeros = _gptq(Xb, W, 128)
    c_o, s_o, z_o, _ = oracle.gptq(X, W, 128)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_o)
    packed = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    q.qg_pack_nibbles(codes, packed)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a16(x_device(Xb[:M].copy(), torch.bfloat16), packed, scales, zeros, Y)
    _status_ok()
    yref, b = oracle.gemm_w4a16_ref(X[:M], oracle.pack_nibbles(c_o), s_o, z_o)
    assert oracle.within_tolerance(bf16_to_f32(u16(Y)), yref, b).all()
    # the method's claim on the calibration batch: a lower layer error than plain rounding
    c0, s0, z0, _ = oracle.quantize_w4_asym(W)
    y_rtn, _ = oracle.gemm_w4a16_ref(X, oracle.pack_nibbles(c0), s0, z0)
    y_gptq, _ = oracle.gemm_w4a16_ref(X, oracle.pack_nibbles(c_o), s_o, z_o)
    exact = oracle.gemm_f64(X, W)
    assert np.sum((exact - y_gptq) ** 2) < 0.8 * np.sum((exact - y_rtn) ** 2)


# ---------------------------------------------------------------------------
# the blocked Cholesky form (qg_gptq_blocked)
# ---------------------------------------------------------------------------
def _gptq_blocked(Xb, W, group):
    q = qlib()
    K, N = W.shape
    codes = torch.full((K, N), 255, dtype=torch.uint8, device="cuda")
    scales = torch.zeros((K // group, N), dtype=torch.int16, device="cuda")
    zeros = torch.full((K // group, N), 255, dtype=torch.uint8, device="cuda")
    q.qg_gptq_blocked(x_device(Xb, torch.bfloat16), cuda(W), codes, scales, zeros, group=group)
    _status_ok()
    return codes.cpu().numpy(), u16(scales), zeros.cpu().numpy()


# a partial last 64-wide panel (K = 296), groups of 8 .. 512 (the 512 case takes the
# narrow column tiling), more columns than one tile
@pytest.mark.parametrize("Mc,K,N,group", [(300, 256, 40, 128), (64, 128, 24, 64), (200, 256, 136, 32),
                                          (17, 384, 8, 128), (100, 296, 40, 8), (160, 1024, 24, 512),
                                          (256, 1024, 200, 128)])
def test_blocked_replay(Mc, K, N, group):
    """The blocked form compensates each row as the sequential definition does, with the
    sums in another order: every code must be the rounding of its teacher-forced replayed
    value up to rounding noise (slack <= 1e-6 grid steps), every scale and zero the
    group's own; and on these well-conditioned cases the codes equal the oracle's except
    where a value sits on a rounding boundary (at most 1 in 1000)."""
    X, Xb = _calib(Mc, K, seed=K + N)
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=N)
    codes, scales, zeros = _gptq_blocked(Xb, W, group)
    slack, sm, zm, st = oracle.gptq_replay(X, W, codes, scales, zeros, group, scale_ulps=0)
    assert st == 0
    assert slack <= 1e-6 and sm == 0 and zm == 0, (slack, sm, zm)
    c_o, s_o, z_o, _ = oracle.gptq(X, W, group)
    assert (codes != c_o).mean() <= 1e-3


def test_blocked_full_size_against_the_sequential_device_path():
    """4096 x 4096 with 512 calibration tokens (the benchmark's GPTQ case).  The sequential
    device path is the oracle's definition bit for bit (test_bitexact); the blocked form
    must give the same codes up to rounding-boundary cases (<= 1e-4 of them), scales
    within one fp16 step and zeros within 1 on every group, and a calibration-batch layer
    error no larger than round-to-nearest's."""
    q = qlib()
    K, N = 4096, 4096
    Mc = synth.CONFIGS["awq"]["calib_tokens"]
    W = synth.workload_weights("w4a16_decode", K, N)
    X, xcb = synth.calibration(K, synth.CONFIGS["awq"])
    Xd, Wd = x_device(xcb, torch.bfloat16), cuda(W)
    outs = []
    for fn in (q.qg_gptq, q.qg_gptq_blocked):
        codes = torch.full((K, N), 255, dtype=torch.uint8, device="cuda")
        scales = torch.zeros((K // 128, N), dtype=torch.int16, device="cuda")
        zeros = torch.full((K // 128, N), 255, dtype=torch.uint8, device="cuda")
        fn(Xd, Wd, codes, scales, zeros)
        _status_ok()
        outs.append((codes.cpu().numpy(), u16(scales), zeros.cpu().numpy()))
    (c_s, s_s, z_s), (c_b, s_b, z_b) = outs
    assert (c_s != c_b).mean() <= 1e-4
    assert np.abs(s_s.astype(np.int32) - s_b.astype(np.int32)).max() <= 1
    assert np.abs(z_s.astype(np.int32) - z_b.astype(np.int32)).max() <= 1
    # layer error on the calibration batch (a sample of 64 tokens)
    Xs = X[:64]
    exact = oracle.gemm_f64(Xs, W)
    c0, s0, z0, _ = oracle.quantize_w4_asym(W)
    y_rtn, _ = oracle.gemm_w4a16_ref(Xs, oracle.pack_nibbles(c0), s0, z0)
    y_b, _ = oracle.gemm_w4a16_ref(Xs, oracle.pack_nibbles(c_b), s_b, z_b)
    assert np.sum((exact - y_b) ** 2) <= np.sum((exact - y_rtn) ** 2)
