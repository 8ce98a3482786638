"""GPU parity: every C-ABI call against the CPU oracle, on the same seeded inputs.

Integers, bytes, packed words, fp16 scales and fp32 token/channel scales must match
bit for bit.  Floating GEMM outputs must satisfy |y - y_ref| <= 1e-2 (|X||W_deq|) + 1e-3
against the oracle's fp64 dot product of the same dequantized operands; the W8A8
output is also bit-exact (its accumulator is exact and its epilogue is two fp32
products).  Shapes are the workloads' own (decode, W8A8, W4A8 in full; prefill on
sampled rows), plus ragged and degenerate cases.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import (bf16_to_f32, cuda, f16_to_f32, quant_w4_asym, quant_w4_sym, sample_rows, u16, u32,
                      x_device)

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


def assert_tol(y, yref, b):
    ok = oracle.within_tolerance(y, yref, b)
    if not ok.all():
        i = np.argwhere(~ok)[0]
        raise AssertionError(f"{(~ok).sum()} elements outside tolerance; first {tuple(i)}: "
                             f"y={y[tuple(i)]} ref={yref[tuple(i)]} bound={b[tuple(i)]}")


def _status_ok():
    q = qlib()
    st = q.qg_device_status()
    assert st == q.QG_OK, q.qg_status_string(st)


# ---------------------------------------------------------------------------
# quantizers (bit-exact)
# ---------------------------------------------------------------------------
# N % 4 == 0 takes the 16-byte kernel (a ragged last CTA at N = 136, 8); N = 30 the
# column-per-thread register kernel
W4_SHAPES = [(1024, 1024, "w4a16_tiny"), (4096, 12288, "w4a16_decode"), (11008, 4096, "w4a16_decode"),
             (384, 136, "w4a16_decode"), (128, 8, "w4a16_decode"), (256, 30, "w4a16_decode")]


@pytest.mark.parametrize("K,N,cfg", W4_SHAPES)
def test_quantize_w4_asym_and_pack_bitexact(K, N, cfg):
    W = synth.workload_weights(cfg, K, N)
    if K == 384:
        W[0:128, 0] = 0.0          # zero group
        W[128:256, 1] = 0.25       # constant group
        W[:, 2] = np.float32(0.5) * np.round(W[:, 2] * 64)  # many exact .5 ties of x/s
        # group range [0, 15 c], c = 2^-8: s = c exactly, z = 0; x / s exactly on (column 3)
        # and 2^-16 beside (column 4) the half-integers j + 1/2
        c = np.float32(2.0 ** -8)
        j = (np.arange(K) % 15).astype(np.float32)
        W[:, 3] = (j + np.float32(0.5)) * c
        W[:, 4] = (j + np.float32(0.5) + np.where(np.arange(K) % 2 == 0, 1, -1).astype(np.float32) * 2.0 ** -16) * c
        W[0::128, 3] = W[0::128, 4] = 0.0
        W[1::128, 3] = W[1::128, 4] = 15 * c
    codes, scales, zeros, packed = quant_w4_asym(W)
    c_o, s_o, z_o, st = oracle.quantize_w4_asym(W)
    assert st == oracle.OK
    _status_ok()
    np.testing.assert_array_equal(codes.cpu().numpy(), c_o)
    np.testing.assert_array_equal(u16(scales), s_o)
    np.testing.assert_array_equal(zeros.cpu().numpy(), z_o)
    np.testing.assert_array_equal(u32(packed), oracle.pack_nibbles(c_o))


def test_smooth_scales_and_w8_channel_bitexact():
    cfg = synth.CONFIGS["w8a8"]
    K, N = cfg["KN"][0]
    W = synth.workload_weights("w8a8", K, N)
    Xc, Xc_bits = synth.calibration(K, cfg)
    q = qlib()
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    inv = torch.empty_like(s)
    q.qg_smooth_scales(x_device(Xc_bits, torch.bfloat16), cuda(W), 0.5, s, inv)
    s_o, inv_o, st = oracle.smooth_scales(Xc, W, 0.5)
    _status_ok()
    np.testing.assert_array_equal(s.cpu().numpy(), s_o)
    np.testing.assert_array_equal(inv.cpu().numpy(), inv_o)
    Wq = torch.empty(K, N, dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    q.qg_quantize_w8_channel(cuda(W), s, Wq, sw)
    Wq_o, sw_o, st = oracle.quantize_w8_channel(W, s_o)
    _status_ok()
    np.testing.assert_array_equal(Wq.cpu().numpy(), Wq_o)
    np.testing.assert_array_equal(sw.cpu().numpy(), sw_o)


@pytest.mark.parametrize("K,N,smooth", [(11008, 4096, True), (16384, 64, False), (2048, 24, True), (100, 136, True),
                                         (4096, 100, True), (20000, 8, False), (6000, 96, True), (700, 64, False),
                                         (8192, 32, True), (4096, 11008, False), (300, 30, True),
                                         (25700, 16, False)])
def test_quantize_w8_channel_shapes_bitexact(K, N, smooth):
    """Both paths of the INT8 channel quantizer: the two-pass kernels over column chunks
    of about 40 MB of W (N % 4 == 0: one chunk at most shapes, 5 at 4096 x 11008 and
    at 11008 x 4096, ragged last chunks and last CTAs) and the general kernel (N % 4 != 0);
    a zero column, and columns whose quotients w / sw sit exactly on and within 2^-16 of
    half-integers (ties to even, and the product form's fallback to the quotient),
    smoothing on and off."""
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=K + N)
    W[:, 3] = 0.0
    if N > 7:
        c = np.float32(2.0 ** -10)  # sw = 127 c / 127 = c exactly
        j = (np.arange(K) % 254 - 127).astype(np.float32)
        W[:, 5] = (j + np.float32(0.5)) * c  # exact ties
        W[:, 6] = (j + np.float32(0.5) + np.where(np.arange(K) % 2 == 0, 1, -1).astype(np.float32) * 2.0 ** -16) * c
        W[0, 5] = W[0, 6] = 127 * c
    s_o = None
    if smooth:
        s_o = np.random.default_rng(K).uniform(0.5, 2.0, K).astype(np.float32)
    q = qlib()
    Wq = torch.empty(K, N, dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    q.qg_quantize_w8_channel(cuda(W), None if s_o is None else cuda(s_o), Wq, sw)
    _status_ok()
    Wq_o, sw_o, _ = oracle.quantize_w8_channel(W, s_o)
    np.testing.assert_array_equal(Wq.cpu().numpy(), Wq_o)
    np.testing.assert_array_equal(sw.cpu().numpy(), sw_o)


@pytest.mark.parametrize("group", [64, 256, 32])
@pytest.mark.parametrize("sym", [False, True])
def test_quantize_w4_other_group_sizes_bitexact(group, sym):
    """Group sizes other than 128 (64 and 256 take the register kernel, 32 the per-column
    kernel), with a ragged column count and smoothing."""
    K, N = 1024, 200
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=group)
    W[0:group, 5] = 0.0                   # zero group
    W[group:2 * group, 7] = 0.01          # constant group
    s_o = np.random.default_rng(group).uniform(0.5, 2.0, K).astype(np.float32)
    if sym:
        codes, scales, packed = quant_w4_sym(W, s_o, group=group)
        c_o, sc_o, _ = oracle.quantize_w4_sym(W, group=group, s_smooth=s_o)
        _status_ok()
        np.testing.assert_array_equal(codes.cpu().numpy().view(np.int8), c_o)
        np.testing.assert_array_equal(scales.cpu().numpy(), sc_o)
    else:
        codes, scales, zeros, packed = quant_w4_asym(W, s_o, group=group)
        c_o, sc_o, z_o, _ = oracle.quantize_w4_asym(W, group=group, s_smooth=s_o)
        _status_ok()
        np.testing.assert_array_equal(codes.cpu().numpy(), c_o)
        np.testing.assert_array_equal(u16(scales), sc_o)
        np.testing.assert_array_equal(zeros.cpu().numpy(), z_o)


def test_quantize_w4_sym_smoothed_bitexact():
    cfg = synth.CONFIGS["w4a8"]
    K, N = cfg["KN"][0]
    W = synth.workload_weights("w4a8", K, N)
    Xc, Xc_bits = synth.calibration(K, cfg)
    s_o, inv_o, _ = oracle.smooth_scales(Xc, W, 0.5)
    codes, scales, packed = quant_w4_sym(W, s_o)
    c_o, sc_o, st = oracle.quantize_w4_sym(W, s_smooth=s_o)
    _status_ok()
    np.testing.assert_array_equal(codes.cpu().numpy().view(np.int8), c_o)
    np.testing.assert_array_equal(scales.cpu().numpy(), sc_o)
    np.testing.assert_array_equal(u32(packed), oracle.pack_nibbles(c_o))


@pytest.mark.parametrize("M,K,chan,mult", [(16, 4096, 8, 50.0), (256, 4096, 8, 50.0), (2048, 4096, 8, 50.0),
                                           (1, 8192, 16, 30.0), (64, 8192, 16, 30.0), (1024, 8192, 16, 30.0),
                                           (3, 136, 2, 10.0)])
def test_smooth_quant_act_i8_bitexact(M, K, chan, mult):
    X, Xb = synth.activations(M, K, "bf16", chan, mult, seed=1)
    X[0, :] = 0.0                       # a zero row -> t = 0, codes 0
    Xb[0, :] = 0
    inv = np.random.default_rng(M).uniform(0.02, 3.0, K).astype(np.float32)
    q = qlib()
    Xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
    t = torch.empty(M, dtype=torch.float32, device="cuda")
    q.qg_smooth_quant_act_i8(x_device(Xb, torch.bfloat16), cuda(inv), Xq, t)
    Xq_o, t_o, _ = oracle.smooth_quant_act_i8(X, inv)
    _status_ok()
    np.testing.assert_array_equal(t.cpu().numpy(), t_o)
    np.testing.assert_array_equal(Xq.cpu().numpy(), Xq_o)
    q.qg_smooth_quant_act_i8(x_device(Xb, torch.bfloat16), None, Xq, t)   # no smoothing
    Xq_o, t_o, _ = oracle.smooth_quant_act_i8(X)
    np.testing.assert_array_equal(t.cpu().numpy(), t_o)
    np.testing.assert_array_equal(Xq.cpu().numpy(), Xq_o)


# ---------------------------------------------------------------------------
# W4A16
# ---------------------------------------------------------------------------
def _w4a16_case(K, N, cfg, Ms, xdtype, rows=None, workspace="auto", repeat=1):
    W = synth.workload_weights(cfg, K, N)
    codes, scales, zeros, packed = quant_w4_asym(W)
    c_o, s_o, z_o, _ = oracle.quantize_w4_asym(W)
    p_o = oracle.pack_nibbles(c_o)
    q = qlib()
    tdt = torch.bfloat16 if xdtype == "bf16" else torch.float16
    for M in Ms:
        X, Xb = synth.activations(M, K, xdtype, seed=M)
        Y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")   # poisoned: every element must be written
        Xd = x_device(Xb, tdt)
        q.qg_gemm_w4a16(Xd, packed, scales, zeros, Y, workspace=workspace)
        _status_ok()
        for _ in range(repeat - 1):   # same inputs, same bits
            Y2 = torch.full_like(Y, float("nan"))
            q.qg_gemm_w4a16(Xd, packed, scales, zeros, Y2, workspace=workspace)
            _status_ok()
            assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))
        r = rows(M) if rows else None
        yref, b = oracle.gemm_w4a16_ref(X, p_o, s_o, z_o, rows=r)
        y = u16(Y)
        y = bf16_to_f32(y) if xdtype == "bf16" else f16_to_f32(y)
        if r is not None:
            y = y[r]
        assert_tol(y, yref, b)


def test_gemm_w4a16_tiny_fp16():
    _w4a16_case(1024, 1024, "w4a16_tiny", [1], "f16")


@pytest.mark.parametrize("K,N", synth.CONFIGS["w4a16_decode"]["KN"])
def test_gemm_w4a16_decode_sweep(K, N):
    _w4a16_case(K, N, "w4a16_decode", synth.CONFIGS["w4a16_decode"]["M"], "bf16")


@pytest.mark.parametrize("K,N", [(4096, 4096), (11008, 4096)])
def test_gemm_w4a16_decode_without_workspace(K, N):
    """The cluster/DSMEM split-K kernel (no workspace) on the same inputs."""
    _w4a16_case(K, N, "w4a16_decode", [1, 16, 32], "bf16", workspace=None)


def test_gemm_w4a16_decode_repeatable():
    """Stream-K finish: calls in a row give identical bits (the split slabs' pieces are summed
    in a fixed order by the CTA that finishes each slab)."""
    _w4a16_case(4096, 12288, "w4a16_decode", [1, 4, 32], "bf16", repeat=3)


def test_gemm_w4a16_workspace_shared_across_shapes():
    """One workspace serves calls of different shapes in turn (its contents never need to
    start at zero)."""
    q = qlib()
    ws = torch.full((q.qg_workspace_size(q.QG_OP_GEMM_W4A16, 32, 4096, 22016),), 0x7F, dtype=torch.uint8, device="cuda")
    for (K, N, M) in [(4096, 12288, 32), (4096, 22016, 1), (4096, 4096, 16), (4096, 22016, 32)]:
        _w4a16_case(K, N, "w4a16_decode", [M], "bf16", workspace=ws)


@pytest.mark.parametrize("xdtype", ["bf16", "f16"])
def test_gemm_w4a16_edge_shapes(xdtype):
    # K = 3 groups, N not a multiple of any tile width, M across every token-tile boundary
    _w4a16_case(384, 136, "w4a16_decode", [1, 2, 3, 5, 7, 8, 9, 17, 31, 33, 63, 65, 127, 129], xdtype)
    _w4a16_case(384, 144, "w4a16_decode", [1, 2, 3, 5, 7, 8, 9, 17, 31, 33, 63, 65, 127, 129], xdtype)  # ragged slab
    _w4a16_case(128, 8, "w4a16_decode", [1, 4], xdtype)
    _w4a16_case(128, 16, "w4a16_decode", [1, 4, 32], xdtype)     # one group, one partial slab
    _w4a16_case(2048, 4096, "w4a16_decode", [3, 12, 27], xdtype)  # fewer units per CTA than a stage


# ---------------------------------------------------------------------------
# W8A8 (SmoothQuant)
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def w8a8_weights():
    cfg = synth.CONFIGS["w8a8"]
    K, N = cfg["KN"][0]
    W = synth.workload_weights("w8a8", K, N)
    Xc, _ = synth.calibration(K, cfg)
    s_o, inv_o, _ = oracle.smooth_scales(Xc, W, 0.5)
    Wq_o, sw_o, _ = oracle.quantize_w8_channel(W, s_o)
    return K, N, inv_o, Wq_o, sw_o


@pytest.mark.parametrize("M,workspace", [(16, "auto"), (256, "auto"), (2048, "auto"), (1, "auto"), (3, "auto"),
                                         (17, "auto"), (16, None), (1, None), (17, None)])
def test_gemm_w8a8_bitexact(M, workspace, w8a8_weights):
    """Below 128 tokens the stream-K kernel (workspace) and the cluster split-K kernel
    (no workspace) both give the oracle's bits."""
    K, N, inv_o, Wq_o, sw_o = w8a8_weights
    X, Xb = synth.workload_activations("w8a8", M, K)
    Xq_o, t_o, _ = oracle.smooth_quant_act_i8(X, inv_o)
    q = qlib()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    q.qg_gemm_w8a8(cuda(Xq_o), cuda(t_o), cuda(Wq_o), cuda(sw_o), Y, acc, workspace=workspace)
    _status_ok()
    rows = sample_rows(M) if M > 256 else None
    acc_o, y_o, yref, b = oracle.gemm_w8a8(Xq_o, t_o, Wq_o, sw_o, rows=rows)
    a = acc.cpu().numpy()
    y = u16(Y)
    if rows is not None:
        a, y = a[rows], y[rows]
    np.testing.assert_array_equal(a, acc_o)
    np.testing.assert_array_equal(y, y_o)
    assert_tol(bf16_to_f32(y), yref, b)
    # without the debug output the result is the same
    Y2 = torch.empty_like(Y)
    q.qg_gemm_w8a8(cuda(Xq_o), cuda(t_o), cuda(Wq_o), cuda(sw_o), Y2, None, workspace=workspace)
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


@pytest.mark.parametrize("K,N", [(512, 144), (1024, 272), (128, 16), (2048, 1296)])
def test_gemm_w8a8_stream_k_edges(K, N):
    """The stream-K kernel across every token tile (16, 32, 64, 128 tokens) and its
    boundaries, on ragged column slabs, one-block K and slabs split between CTAs; the
    workspace starts with garbage (its contents must not matter)."""
    rng = np.random.default_rng(K + N)
    q = qlib()
    ws = torch.full((q.qg_workspace_size(q.QG_OP_GEMM_W8A8, 127, K, N),), 0x5A, dtype=torch.uint8, device="cuda")
    for M in [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 127]:
        Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        Wq = rng.integers(-127, 128, (K, N)).astype(np.int8)
        t = rng.uniform(0.01, 1.0, M).astype(np.float32)
        sw = rng.uniform(0.001, 0.01, N).astype(np.float32)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        acc = torch.full((M, N), -1, dtype=torch.int32, device="cuda")
        q.qg_gemm_w8a8(cuda(Xq), cuda(t), cuda(Wq), cuda(sw), Y, acc, workspace=ws)
        _status_ok()
        acc_o, y_o, _, _ = oracle.gemm_w8a8(Xq, t, Wq, sw)
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o, err_msg=f"M={M}")
        np.testing.assert_array_equal(u16(Y), y_o, err_msg=f"M={M}")


# ---------------------------------------------------------------------------
# W4A8
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def w4a8_weights():
    cfg = synth.CONFIGS["w4a8"]
    K, N = cfg["KN"][0]
    W = synth.workload_weights("w4a8", K, N)
    Xc, _ = synth.calibration(K, cfg)
    s_o, inv_o, _ = oracle.smooth_scales(Xc, W, 0.5)
    c_o, sc_o, _ = oracle.quantize_w4_sym(W, s_smooth=s_o)
    return K, N, inv_o, oracle.pack_nibbles(c_o), sc_o


@pytest.mark.parametrize("workspace", ["auto", None])
@pytest.mark.parametrize("M", [1, 64, 1024, 3, 33])
def test_gemm_w4a8(M, workspace, w4a8_weights):
    """17..127 tokens: the stream-K kernel with a workspace, the cluster split-K kernel
    without one; 16 tokens and fewer: split-K either way; 1024 tokens: the tile kernel."""
    K, N, inv_o, p_o, sc_o = w4a8_weights
    X, Xb = synth.workload_activations("w4a8", M, K)
    Xq_o, t_o, _ = oracle.smooth_quant_act_i8(X, inv_o)
    q = qlib()
    G = K // 128
    want_part = M <= 64
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    part = torch.empty(M, G, N, dtype=torch.int32, device="cuda") if want_part else None
    q.qg_gemm_w4a8(cuda(Xq_o), cuda(t_o), cuda(p_o.view(np.int32)), cuda(sc_o), Y, part, workspace=workspace)
    _status_ok()
    rows = sample_rows(M) if M > 64 else None
    part_o, yref, b = oracle.gemm_w4a8(Xq_o, t_o, p_o, sc_o, rows=rows, want_part=want_part)
    if want_part:
        np.testing.assert_array_equal(part.cpu().numpy(), part_o)
    y = bf16_to_f32(u16(Y))
    if rows is not None:
        y = y[rows]
    assert_tol(y, yref, b)


@pytest.mark.parametrize("K,N", [(512, 144), (1024, 272), (128, 16), (2048, 1296)])
def test_gemm_w4a8_stream_k_edges(K, N):
    """The W4A8 stream-K kernel (17..127 tokens) across its token tiles (32, 64 and chunks
    of 64 with ragged last chunks), ragged column slabs, one-group K and slabs split
    between CTAs, plus the split-K kernel the same call takes at 16 tokens and fewer; the
    workspace starts with garbage (its contents must not matter)."""
    rng = np.random.default_rng(3 * K + N)
    q = qlib()
    G = K // 128
    ws = torch.full((q.qg_workspace_size(q.QG_OP_GEMM_W4A8, 127, K, N),), 0x5A, dtype=torch.uint8, device="cuda")
    codes = rng.integers(-7, 8, (K, N)).astype(np.int8)
    sg = rng.uniform(0.001, 0.01, (G, N)).astype(np.float32)
    p_o = oracle.pack_nibbles(codes)
    for M in [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 127]:
        Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        t = rng.uniform(0.01, 1.0, M).astype(np.float32)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        part = torch.full((M, G, N), -1, dtype=torch.int32, device="cuda")
        q.qg_gemm_w4a8(cuda(Xq), cuda(t), cuda(p_o.view(np.int32)), cuda(sg), Y, part, workspace=ws)
        _status_ok()
        part_o, yref, b = oracle.gemm_w4a8(Xq, t, p_o, sg)
        np.testing.assert_array_equal(part.cpu().numpy(), part_o, err_msg=f"M={M}")
        assert_tol(bf16_to_f32(u16(Y)), yref, b)
        # without the debug output the same kernel path gives the same Y
        Y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        q.qg_gemm_w4a8(cuda(Xq), cuda(t), cuda(p_o.view(np.int32)), cuda(sg), Y2, None, workspace=ws)
        _status_ok()
        assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16)), f"M={M}"


# ---------------------------------------------------------------------------
# status word: bounded waits and non-finite inputs
# ---------------------------------------------------------------------------
def test_bounded_wait_gives_up_and_device_stays_usable():
    q = qlib()
    q.qg_selftest_bounded_wait(2_000_000)   # 2 ms limit; the wait can never complete
    assert q.qg_device_status() == q.QG_ERR_TIMEOUT
    assert q.qg_device_status() == q.QG_OK  # cleared on read
    test_gemm_w4a16_tiny_fp16()             # the context still works


def test_nonfinite_weights_reported():
    q = qlib()
    W = synth.weights(256, 64, 0.02)
    W[3, 5] = np.inf
    quant_w4_asym(W)
    assert q.qg_device_status() == q.QG_ERR_NONFINITE
    W = synth.weights(256, 64, 0.02)
    W[0, 0], W[1, 0] = 1e6, -1e6            # scale 2e6/15 does not fit fp16
    quant_w4_asym(W)
    assert q.qg_device_status() == q.QG_ERR_RANGE


# ---------------------------------------------------------------------------
# prefill W4A16 at full size: every 64th row plus the first and the last, across all N
# (every 256-token tile of the tile kernel is visited four times; oracle cost bounded)
# ---------------------------------------------------------------------------
def rows_every_64(M):
    return np.array(sorted(set(range(0, M, 64)) | {0, M - 1}), np.int64)


@pytest.mark.parametrize("K,N", synth.CONFIGS["w4a16_prefill"]["KN"])
def test_gemm_w4a16_prefill_sampled(K, N):
    _w4a16_case(K, N, "w4a16_prefill", [4096, 8192], "bf16", rows=rows_every_64)


# ---------------------------------------------------------------------------
# tensor-memory tile kernels (M >= 128) on ragged shapes: partial M and N tiles
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,N", [(128, 256, 208), (130, 384, 144), (257, 256, 272), (300, 512, 400)])
def test_tile_w8a8_ragged(M, K, N):
    rng = np.random.default_rng(M + N)
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    Wq = rng.integers(-127, 128, (K, N)).astype(np.int8)
    t = rng.uniform(0.01, 1.0, M).astype(np.float32)
    sw = rng.uniform(0.001, 0.01, N).astype(np.float32)
    q = qlib()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    acc = torch.full((M, N), -1, dtype=torch.int32, device="cuda")
    q.qg_gemm_w8a8(cuda(Xq), cuda(t), cuda(Wq), cuda(sw), Y, acc)
    _status_ok()
    acc_o, y_o, yref, b = oracle.gemm_w8a8(Xq, t, Wq, sw)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    np.testing.assert_array_equal(u16(Y), y_o)


@pytest.mark.parametrize("M,K,N", [(128, 256, 208), (130, 384, 144), (257, 256, 272), (300, 512, 400)])
def test_tile_w4a8_ragged(M, K, N):
    rng = np.random.default_rng(M * N)
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    codes = rng.integers(-7, 8, (K, N)).astype(np.int8)
    sg = rng.uniform(0.001, 0.01, (K // 128, N)).astype(np.float32)
    t = rng.uniform(0.01, 1.0, M).astype(np.float32)
    p_o = oracle.pack_nibbles(codes)
    q = qlib()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    part = torch.full((M, K // 128, N), -1, dtype=torch.int32, device="cuda")
    q.qg_gemm_w4a8(cuda(Xq), cuda(t), cuda(p_o.view(np.int32)), cuda(sg), Y, part)
    _status_ok()
    part_o, yref, b = oracle.gemm_w4a8(Xq, t, p_o, sg)
    np.testing.assert_array_equal(part.cpu().numpy(), part_o)
    assert_tol(bf16_to_f32(u16(Y)), yref, b)


@pytest.mark.parametrize("M,K,N", [(128, 256, 208), (130, 384, 144), (257, 256, 272), (513, 512, 400)])
def test_tile_w4a16_ragged(M, K, N):
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=M)
    codes, scales, zeros, packed = quant_w4_asym(W)
    c_o, s_o, z_o, _ = oracle.quantize_w4_asym(W)
    X, Xb = synth.activations(M, K, "bf16", seed=N)
    q = qlib()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a16(x_device(Xb, torch.bfloat16), packed, scales, zeros, Y)
    _status_ok()
    yref, b = oracle.gemm_w4a16_ref(X, oracle.pack_nibbles(c_o), s_o, z_o)
    assert_tol(bf16_to_f32(u16(Y)), yref, b)
