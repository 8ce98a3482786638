"""GPU parity of the INT8 outlier side path ("LLM inference cost: W8A8/W4A8 ...", sec. 2.2,
second technique) against the CPU oracle, through the C ABI.

Bit-exact: the split (outlier offsets, INT8 codes, fp32 scales, the dense remainder)
and, through the ordinary INT4 quantizer, the dense part's codes.  Within the stated
tolerance |y - y_ref| <= 1e-2 (|X||W|) + 1e-3: the layer output with the side path,
against the oracle's binary64 product of the same dequantized operands (the side path
adds its fp32 sum to the rounded INT4 output and rounds once more: 2^-9 |y| each time).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_f32, cuda, f16_to_f32, quant_w4_asym, u16, x_device

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


def _split(W, s=None, group=128, count=3):
    q = qlib()
    K, N = W.shape
    G = K // group
    idx = torch.full((G, count, N), 255, dtype=torch.uint8, device="cuda")
    c8 = torch.zeros((G, count, N), dtype=torch.int8, device="cuda")
    s8 = torch.full((G, N), float("nan"), dtype=torch.float32, device="cuda")
    dense = torch.full((K, N), float("nan"), dtype=torch.float32, device="cuda")
    q.qg_outlier_split_w4(cuda(W), None if s is None else cuda(s), group, count, idx, c8, s8, dense)
    _status_ok()
    return idx, c8, s8, dense


def _check_split(W, s=None, group=128, count=3):
    idx, c8, s8, dense = _split(W, s, group, count)
    i_o, c_o, s_o, d_o, st = oracle.outlier_split(W, group=group, count=count, s_smooth=s)
    assert st == 0
    np.testing.assert_array_equal(idx.cpu().numpy(), i_o)
    np.testing.assert_array_equal(c8.cpu().numpy(), c_o)
    np.testing.assert_array_equal(s8.cpu().numpy(), s_o)
    np.testing.assert_array_equal(dense.cpu().numpy().view(np.uint32), d_o.view(np.uint32))
    return idx, c8, s8, dense, (i_o, c_o, s_o, d_o)


def test_split_bitexact_on_the_decode_weight():
    K, N = 4096, 12288
    W = synth.workload_weights("w4a16_decode", K, N)
    _check_split(W)


@pytest.mark.parametrize("group,count", [(128, 3), (64, 2), (256, 6), (128, 8), (128, 0)])
def test_split_ragged_ties_and_smoothing(group, count):
    K, N = 768, 40
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=group + count)
    W[5, 0] = W[9, 0] = 2.0            # ties on |w|: the smaller k ranks first
    W[130, 1], W[140, 1] = -3.0, 3.0
    W[256:384, 2] = 0.0                # an all-zero group: s8 = 0, codes 0
    s = np.random.default_rng(1).uniform(0.5, 2.0, K).astype(np.float32)
    _check_split(W, None, group, count)
    _check_split(W, s, group, count)


@pytest.mark.parametrize("M,xdt", [(1, "bf16"), (4, "bf16"), (32, "bf16"), (160, "bf16"), (3, "f16")])
def test_layer_with_side_path(M, xdt):
    q = qlib()
    K, N = 1024, 384
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=M)
    idx, c8, s8, dense, (i_o, c_o, s_o, d_o) = _check_split(W)
    codes, scales, zeros, packed = quant_w4_asym(d_o)
    c_ref, sc_ref, z_ref, _ = oracle.quantize_w4_asym(d_o)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    X, Xb = synth.activations(M, K, xdt, seed=M)
    dt = torch.bfloat16 if xdt == "bf16" else torch.float16
    Y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    q.qg_gemm_w4a16_outlier(x_device(Xb, dt), packed, scales, zeros, idx, c8, s8, Y)
    _status_ok()
    y = (bf16_to_f32 if xdt == "bf16" else f16_to_f32)(u16(Y))
    yref, b = oracle.gemm_w4a16_outlier_ref(X, oracle.pack_nibbles(c_ref), sc_ref, z_ref, i_o, c_o, s_o)
    ok = oracle.within_tolerance(y, yref, b)
    assert ok.all(), f"{(~ok).sum()} outside tolerance"
    # the side path matters: without it the same outputs miss the outliers' share
    Y0 = torch.empty_like(Y)
    q.qg_gemm_w4a16(x_device(Xb, dt), packed, scales, zeros, Y0)
    _status_ok()
    y0 = (bf16_to_f32 if xdt == "bf16" else f16_to_f32)(u16(Y0))
    assert np.abs(y - yref).sum() < 0.5 * np.abs(y0 - yref).sum()


# ---------------------------------------------------------------------------
# the side path fused into the decode kernel (workspace given, 1..4 outliers, M < 128):
# the side sums join each slab piece's fp32 tile, so Y is rounded once
# ---------------------------------------------------------------------------
def _exact_side(K, N, count, seed):
    """Exact operands: INT4 codes with power-of-two scales, and `count` distinct offsets per
    group and column with INT8 codes |c| <= 15 and power-of-two scales 2^-2..2^0, so every
    product and partial sum of the layer is exact in binary32."""
    G = K // 128
    r = synth.rng(seed, synth.S_EXACT, 7, K, N)
    idx = np.argsort(r.random((G, 128, N)), axis=1)[:, :count, :].astype(np.uint8)
    c8 = r.integers(-15, 16, (G, count, N)).astype(np.int8)
    s8 = np.ldexp(1.0, r.integers(-2, 1, (G, N))).astype(np.float32)
    return idx, c8, s8


@pytest.mark.parametrize("M,count,N", [(1, 3, 12288), (16, 3, 12288), (5, 1, 384), (27, 4, 1024), (40, 2, 256)])
def test_fused_side_path_exact(M, count, N):
    q = qlib()
    K = 4096 if N == 12288 else 1024
    codes, scales, zeros = synth.exact_w4_asym(K, N, seed=M)
    packed = oracle.pack_nibbles(codes)
    idx, c8, s8 = _exact_side(K, N, count, seed=M + count)
    X, Xb = synth.exact_activations(M, K, seed=M)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a16_outlier(x_device(Xb, torch.bfloat16), cuda(packed.view(np.int32)), cuda(scales.view(np.int16)),
                            cuda(zeros), cuda(idx), cuda(c8), cuda(s8), Y)
    _status_ok()
    yref, _ = oracle.gemm_w4a16_outlier_ref(X, packed, scales, zeros, idx, c8, s8)
    y32 = yref.astype(np.float32)
    assert np.array_equal(y32.astype(np.float64), yref), "operands are not an exact case"
    want = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = u16(Y)
    bad = got != want
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ (M={M}, count={count}, N={N})"


@pytest.mark.parametrize("M", [1, 16])
@pytest.mark.parametrize("workspace", ["auto", None])
def test_layer_decode_width(M, workspace):
    """The decode layer's full 4096 x 12288 weight, fused (workspace) and two-step (none)."""
    q = qlib()
    K, N = 4096, 12288
    W = synth.workload_weights("w4a16_decode", K, N)
    idx, c8, s8, dense, (i_o, c_o, s_o, d_o) = _check_split(W)
    codes, scales, zeros, packed = quant_w4_asym(d_o)
    c_ref, sc_ref, z_ref, _ = oracle.quantize_w4_asym(d_o)
    X, Xb = synth.activations(M, K, "bf16", seed=M)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a16_outlier(x_device(Xb, torch.bfloat16), packed, scales, zeros, idx, c8, s8, Y, workspace=workspace)
    _status_ok()
    yref, b = oracle.gemm_w4a16_outlier_ref(X, oracle.pack_nibbles(c_ref), sc_ref, z_ref, i_o, c_o, s_o)
    ok = oracle.within_tolerance(bf16_to_f32(u16(Y)), yref, b)
    assert ok.all(), f"{(~ok).sum()} outside tolerance"


def test_fused_offset_out_of_range_is_reported():
    """An offset past the group is skipped and reported (QG_ERR_RANGE); no read past X."""
    q = qlib()
    K, N, M = 1024, 256, 2
    codes, scales, zeros = synth.exact_w4_asym(K, N, seed=1)
    packed = oracle.pack_nibbles(codes)
    idx, c8, s8 = _exact_side(K, N, 3, seed=1)
    idx[2, 1, 7] = 200
    _, Xb = synth.exact_activations(M, K, seed=1)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a16_outlier(x_device(Xb, torch.bfloat16), cuda(packed.view(np.int32)), cuda(scales.view(np.int16)),
                            cuda(zeros), cuda(idx), cuda(c8), cuda(s8), Y)
    assert q.qg_device_status() == q.QG_ERR_RANGE
