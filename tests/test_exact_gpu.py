"""GPU parity on exact-arithmetic operands: every float GEMM kernel, bit for bit.

On operands drawn as INT4 codes with power-of-two scales and small integer
activations (``synth.exact_*``), every product and every partial sum of the
quantized GEMMs is an integer multiple of the smallest scale below 2^24 of it, so it
is exact in binary32 whatever the summation order, blocking or split.  A correct
kernel therefore returns the exact product Y = X * dequant(W) ("AI Infra guide, ch.4
Quantization", sec. 3.1) rounded once to the output dtype, and the oracle's binary64
result, rounded once, is that value.  Unlike the tolerance band of the general
parity tests, this catches a fault confined to one group, one slab piece or one
reduction slot.

Bounds behind the exactness (units of the smallest scale 2^-2):
* W4A16: |x| <= 8, |q - z| <= 15, scales 2^e, e in [-2, 0]: one term <= 480, so any
  partial sum over K <= 28672 stays below 13.8e6 < 2^24; the decode kernel's raw
  group sums sum x (128 + q) <= 128 * 8 * 143 are exact too.
* W4A8: |qx| <= 31, |q| <= 7, group scales 2^e, e in [-2, 0], token scales 2^f: one
  group partial <= 27776, so sum_g P s_g over K <= 8192 stays below 7.2e6 < 2^24.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import cuda, u16, x_device

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


def rows_every_64(M):
    """Every 64th row plus the first and the last."""
    return np.array(sorted(set(range(0, M, 64)) | {0, M - 1}), np.int64)


def expected_bits(yref, dtype):
    """The exact binary64 result rounded once to the output dtype (exact in binary32 first)."""
    y32 = yref.astype(np.float32)
    assert np.array_equal(y32.astype(np.float64), yref), "operands are not an exact case"
    t = torch.from_numpy(y32)
    t16 = t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float16)
    return t16.view(torch.int16).numpy().view(np.uint16)


def assert_bits(got, want, what):
    bad = got != want
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outputs differ; first at {i}: "
                             f"got 0x{int(got[i]):04x} want 0x{int(want[i]):04x}")


def w4a16_exact_operands(K, N, seed=0):
    codes, scales, zeros = synth.exact_w4_asym(K, N, seed=seed)
    packed = oracle.pack_nibbles(codes)
    q = qlib()
    # the device packs the same codes itself (a2 is bit-exact): the two sides share no packing
    pd = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    q.qg_pack_nibbles(cuda(codes), pd)
    assert np.array_equal(pd.cpu().numpy().view(np.uint32), packed)
    return codes, scales, zeros, packed, pd, cuda(scales.view(np.int16)), cuda(zeros)


def run_w4a16(Xb, dtype, pd, sd, zd, N, workspace):
    q = qlib()
    M = Xb.shape[0]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    Y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
    q.qg_gemm_w4a16(x_device(Xb, tdt), pd, sd, zd, Y, workspace=workspace)
    st = q.qg_device_status()
    assert st == q.QG_OK, q.qg_status_string(st)
    return u16(Y)


# ---------------------------------------------------------------------------
# W4A16 decode (stream-K kernel with a workspace) and the no-workspace kernel
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("K,N", [(4096, 22016), (11008, 4096), (4096, 12288), (384, 136)])
@pytest.mark.parametrize("M", [1, 4, 16, 32, 45])
@pytest.mark.parametrize("workspace", ["auto", None])
def test_w4a16_decode_exact(K, N, M, workspace):
    if workspace is None and M > 16 and K * N > 4096 * 12288:
        pytest.skip("the no-workspace kernel is covered at this M on the smaller shapes")
    _, scales, zeros, packed, pd, sd, zd = w4a16_exact_operands(K, N, seed=M)
    X, Xb = synth.exact_activations(M, K, seed=M)
    got = run_w4a16(Xb, "bf16", pd, sd, zd, N, workspace)
    yref, _ = oracle.gemm_w4a16_ref(X, packed, scales, zeros)
    assert_bits(got, expected_bits(yref, "bf16"), f"W4A16 M={M} K={K} N={N} workspace={workspace}")


@pytest.mark.parametrize("M", [1, 5])
@pytest.mark.parametrize("workspace", ["auto", None])
def test_w4a16_fp16_exact(M, workspace):
    K, N = 1024, 1024
    _, scales, zeros, packed, pd, sd, zd = w4a16_exact_operands(K, N, seed=3)
    X, Xb = synth.exact_activations(M, K, dtype="f16", seed=3)
    got = run_w4a16(Xb, "f16", pd, sd, zd, N, workspace)
    yref, _ = oracle.gemm_w4a16_ref(X, packed, scales, zeros)
    assert_bits(got, expected_bits(yref, "f16"), f"W4A16 fp16 M={M}")


# ---------------------------------------------------------------------------
# W4A16 prefill (tcgen05 tile kernel), full prefill widths and ragged tiles
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,N", [(4096, 8192, 28672), (4096, 28672, 8192), (128, 8192, 28672), (300, 384, 136)])
def test_w4a16_prefill_exact(M, K, N):
    _, scales, zeros, packed, pd, sd, zd = w4a16_exact_operands(K, N, seed=11)
    X, Xb = synth.exact_activations(M, K, seed=11)
    got = run_w4a16(Xb, "bf16", pd, sd, zd, N, "auto")
    rows = rows_every_64(M)
    yref, _ = oracle.gemm_w4a16_ref(X, packed, scales, zeros, rows=rows)
    assert_bits(got[rows], expected_bits(yref, "bf16"), f"W4A16 prefill M={M} K={K} N={N}")


# ---------------------------------------------------------------------------
# W4A8: the cluster kernel (M <= 16), the stream-K kernel (17..127, with a workspace)
# and the tile kernel (M >= 128), against the oracle's output definition
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M", [1, 3, 16, 17, 64, 100, 128, 1024])
@pytest.mark.parametrize("workspace", ["auto", None])
def test_w4a8_exact(M, workspace):
    # without a workspace, 17..127 tokens take the cluster kernel in chunks
    K, N = 8192, 8192
    codes, sg = synth.exact_w4_sym(K, N, seed=5)
    packed = oracle.pack_nibbles(codes)
    Xq, t = synth.exact_act_i8(M, K, seed=M)
    q = qlib()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a8(cuda(Xq), cuda(t), cuda(packed.view(np.int32)), cuda(sg), Y, None, workspace=workspace)
    st = q.qg_device_status()
    assert st == q.QG_OK, q.qg_status_string(st)
    rows = rows_every_64(M) if M > 128 else None
    _, yref, _, y_o = oracle.gemm_w4a8(Xq, t, packed, sg, rows=rows, want_part=False, want_y=True)
    want = expected_bits(yref, "bf16")
    assert np.array_equal(y_o, want)   # the output definition, exact here
    got = u16(Y)
    assert_bits(got if rows is None else got[rows], want, f"W4A8 M={M} workspace={workspace}")


# ---------------------------------------------------------------------------
# 2:4 sparse INT4
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M", [1, 4, 17, 32, 45])
@pytest.mark.parametrize("tc", [False, True])
def test_w4a16_24_exact(M, tc):
    """Both 2:4 GEMMs: the SIMT kernel on the canonical layout and the mma.sp decode
    kernel on the tensor-core layout (qg_pack24_tc), on a full decode width."""
    K, N = 4096, 1024 if not tc else 12288
    if not tc and M > 17:
        pytest.skip("the SIMT kernel is covered at M <= 17")
    codes, scales, zeros = synth.exact_w4_asym(K, N, seed=9)
    # a 2:4 pattern along K: two positions per block of four, drawn at random; the
    # oracle's pruning keeps exactly them (kept magnitudes 2..3, dropped 0..1)
    r = synth.rng(9, synth.S_EXACT, 5, K, N)
    keys = r.random((K // 4, 4, N))
    keep = np.argsort(keys, axis=1)[:, :2, :]
    mag = r.uniform(0.0, 1.0, (K // 4, 4, N)).astype(np.float32)
    np.put_along_axis(mag, keep, r.uniform(2.0, 3.0, (K // 4, 2, N)).astype(np.float32), axis=1)
    Wpat = mag.reshape(K, N)
    _, meta = oracle.prune24(Wpat)
    vals = oracle.pack24_vals(codes, meta)
    X, Xb = synth.exact_activations(M, K, seed=M)
    q = qlib()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    vd = cuda(vals.view(np.int32))
    if tc:
        vt = torch.full_like(vd, -1)
        q.qg_pack24_tc(vd, vt)
        q.qg_gemm_w4a16_24_tc(x_device(Xb, torch.bfloat16), vt, cuda(meta.view(np.int32)),
                              cuda(scales.view(np.int16)), cuda(zeros), Y)
    else:
        q.qg_gemm_w4a16_24(x_device(Xb, torch.bfloat16), vd, cuda(meta.view(np.int32)),
                           cuda(scales.view(np.int16)), cuda(zeros), Y)
    st = q.qg_device_status()
    assert st == q.QG_OK, q.qg_status_string(st)
    yref, _ = oracle.gemm_w4a16_24_ref(X, vals, meta, scales, zeros)
    assert_bits(u16(Y), expected_bits(yref, "bf16"), f"2:4 M={M} tc={tc}")
