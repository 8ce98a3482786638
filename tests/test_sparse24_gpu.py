"""GPU parity of 2:4 structured sparsity + INT4 ("LLM inference cost: W8A8/W4A8 ...",
sec. 3.2) against the CPU oracle, through the C ABI.

Bit-exact: the pruned matrix and its position words, the INT4 codes of the pruned matrix
(the ordinary quantizer) and the packed kept codes.  Within the stated tolerance
|y - y_ref| <= 1e-2 (|X||W|) + 1e-3: the GEMM against the oracle's binary64 product of the
same dequantized sparse operand (fp32 accumulation, one rounding to the output dtype).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_f32, cuda, f16_to_f32, u16, x_device

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


def _sparse_weights(W):
    """Prune, quantize and pack on the device; compare every stored array with the oracle."""
    q = qlib()
    K, N = W.shape
    Wd = cuda(W)
    Wp = torch.full((K, N), float("nan"), dtype=torch.float32, device="cuda")
    meta = torch.zeros((K // 32, N), dtype=torch.int32, device="cuda")
    q.qg_prune24(Wd, Wp, meta)
    _status_ok()
    Wp_o, meta_o = oracle.prune24(W)
    np.testing.assert_array_equal(Wp.cpu().numpy().view(np.uint32), Wp_o.view(np.uint32))
    np.testing.assert_array_equal(meta.cpu().numpy().view(np.uint32), meta_o)
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    scales = torch.empty(K // 128, N, dtype=torch.int16, device="cuda")
    zeros = torch.empty(K // 128, N, dtype=torch.uint8, device="cuda")
    q.qg_quantize_w4_group(Wp, None, 128, False, codes, scales, zeros)
    vals = torch.zeros((K // 16, N), dtype=torch.int32, device="cuda")
    q.qg_pack24_vals(codes, meta, vals)
    _status_ok()
    c_o, s_o, z_o, _ = oracle.quantize_w4_asym(Wp_o)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_o)
    vals_o = oracle.pack24_vals(c_o, meta_o)
    np.testing.assert_array_equal(vals.cpu().numpy().view(np.uint32), vals_o)
    return (vals, meta, scales, zeros), (vals_o, meta_o, s_o, z_o)


def test_prune_pack_bitexact_on_the_decode_weight():
    K, N = 4096, 12288
    _sparse_weights(synth.workload_weights("w4a16_decode", K, N))


def test_prune_ties_and_zero_blocks():
    K, N = 256, 40
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=11)
    W[8:12, 0] = [0.5, -0.5, 0.5, 0.1]
    W[20:24, 1] = 0.0
    W[32:36, 2] = [-1.0, 1.0, -1.0, 1.0]
    _sparse_weights(W)


@pytest.mark.parametrize("M,N,xdt", [(1, 12288, "bf16"), (4, 384, "bf16"), (17, 136, "bf16"), (64, 256, "bf16"),
                                     (3, 200, "f16")])
def test_gemm_within_tolerance(M, N, xdt):
    q = qlib()
    K = 4096 if N == 12288 else 512
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=M + N)
    dev, ref = _sparse_weights(W)
    X, Xb = synth.activations(M, K, xdt, seed=M)
    dt = torch.bfloat16 if xdt == "bf16" else torch.float16
    Y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    q.qg_gemm_w4a16_24(x_device(Xb, dt), *dev, Y)
    _status_ok()
    y = (bf16_to_f32 if xdt == "bf16" else f16_to_f32)(u16(Y))
    yref, b = oracle.gemm_w4a16_24_ref(X, *ref)
    ok = oracle.within_tolerance(y, yref, b)
    assert ok.all(), f"{(~ok).sum()} outside tolerance"


# ---------------------------------------------------------------------------
# the tensor-core form: qg_pack24_tc + qg_gemm_w4a16_24_tc (mma.sp decode kernel)
# ---------------------------------------------------------------------------
def _tc_layout(vals):
    """The documented tensor-core layout, restated here from its definition in the header:
    word u = 2t + hb of group gq holds, for step s, block 8s + t + 4hb's first kept code at
    bits 4s and its second at bits 16 + 4s."""
    K16, N = vals.shape
    out = np.zeros_like(vals)
    for gq in range(K16 // 8):
        v = vals[8 * gq:8 * gq + 8].astype(np.uint64)
        for u in range(8):
            t, hb = u >> 1, u & 1
            w = np.zeros(N, np.uint64)
            for s in range(4):
                bl = 8 * s + t + 4 * hb
                byte = (v[bl >> 2] >> np.uint64(8 * (bl & 3))) & np.uint64(0xFF)
                w |= (byte & np.uint64(0xF)) << np.uint64(4 * s)
                w |= (byte >> np.uint64(4)) << np.uint64(16 + 4 * s)
            out[8 * gq + u] = w.astype(np.uint32)
    return out


def _tc_operands(vals):
    q = qlib()
    vals_tc = torch.full_like(vals, -1)
    q.qg_pack24_tc(vals, vals_tc)
    _status_ok()
    np.testing.assert_array_equal(vals_tc.cpu().numpy().view(np.uint32), _tc_layout(vals.cpu().numpy().view(np.uint32)))
    return vals_tc


@pytest.mark.parametrize("M,N,xdt", [(1, 12288, "bf16"), (16, 12288, "bf16"), (4, 384, "bf16"), (17, 160, "bf16"),
                                     (32, 256, "bf16"), (45, 96, "bf16"), (3, 224, "f16")])
def test_tc_gemm_within_tolerance(M, N, xdt):
    q = qlib()
    K = 4096 if N == 12288 else 512
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=M + N + 1)
    (vals, meta, scales, zeros), ref = _sparse_weights(W)
    vals_tc = _tc_operands(vals)
    X, Xb = synth.activations(M, K, xdt, seed=M)
    dt = torch.bfloat16 if xdt == "bf16" else torch.float16
    Y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    q.qg_gemm_w4a16_24_tc(x_device(Xb, dt), vals_tc, meta, scales, zeros, Y)
    _status_ok()
    y = (bf16_to_f32 if xdt == "bf16" else f16_to_f32)(u16(Y))
    yref, b = oracle.gemm_w4a16_24_ref(X, *ref)
    ok = oracle.within_tolerance(y, yref, b)
    assert ok.all(), f"{(~ok).sum()} outside tolerance"


def test_tc_repeat_calls_identical():
    q = qlib()
    K, N, M = 4096, 12288, 4
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=3)
    (vals, meta, scales, zeros), _ = _sparse_weights(W)
    vals_tc = _tc_operands(vals)
    _, Xb = synth.activations(M, K, "bf16", seed=3)
    Xd = x_device(Xb, torch.bfloat16)
    outs = []
    for _ in range(3):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        q.qg_gemm_w4a16_24_tc(Xd, vals_tc, meta, scales, zeros, Y)
        outs.append(u16(Y))
    _status_ok()
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
