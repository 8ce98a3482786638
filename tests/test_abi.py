"""The C-ABI library loads, exports every entry point include/qgemm.h declares, and
rejects bad arguments before launching anything.  CPU only: every call here fails
validation, so no CUDA call is reached."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemm.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ["qg_quantize_w4_group", "qg_pack_nibbles", "qg_gemm_w4a16", "qg_smooth_quant_act_i8",
                 "qg_gemm_w8a8", "qg_gemm_w4a8", "qg_smooth_scales", "qg_quantize_w8_channel", "qg_device_status",
                 "qg_status_string", "qg_awq_act_mean", "qg_awq_scales", "qg_awq_scale_act", "qg_awq_search",
                 "qg_outlier_split_w4", "qg_outlier_side_add", "qg_gemm_w4a16_outlier", "qg_prune24",
                 "qg_pack24_vals", "qg_gemm_w4a16_24", "qg_gptq"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    import bit_quantized_gemm_group_b200 as q
    L = q.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert set(q.EXPORTS) >= set(declared_symbols())


def test_status_strings():
    import bit_quantized_gemm_group_b200 as q
    for code, name in q.STATUS.items():
        assert q.qg_status_string(code) == name


P = ctypes.c_void_p
A = P(0x10000)        # aligned fake device address (never dereferenced: validation fails first)
B = P(0x10008)        # 8-byte but not 16-byte aligned


@pytest.mark.parametrize("args,want", [
    # quantize_w4_group(W, s, K, N, group, sym, codes, scales, zeros, stream)
    ((None, None, 256, 64, 128, 0, A, A, A, None), 1),
    ((A, None, 256, 64, 128, 0, A, A, None, None), 1),       # asym needs zeros
    ((A, None, 256, 64, 128, 1, A, A, A, None), 1),          # sym takes no zeros
    ((A, None, 200, 64, 128, 0, A, A, A, None), 2),          # K % group
    ((A, None, 256, 64, 12, 0, A, A, A, None), 2),           # group % 8
    ((A, None, 256, 0, 128, 0, A, A, A, None), 2),
    ((B, None, 256, 64, 128, 0, A, A, A, None), 3),
])
def test_quantize_rejects(args, want):
    import bit_quantized_gemm_group_b200 as q
    assert q.lib().qg_quantize_w4_group(*args) == want


@pytest.mark.parametrize("args,want", [
    # gemm_w4a16(X, xdt, M, K, N, packed, scales, zeros, group, Y, ws, ws_bytes, stream)
    ((A, 7, 1, 256, 64, A, A, A, 128, A, None, 0, None), 4),
    ((A, 1, 1, 200, 64, A, A, A, 128, A, None, 0, None), 2),
    ((A, 1, 1, 256, 60, A, A, A, 128, A, None, 0, None), 2),
    ((A, 1, 1, 256, 64, A, A, A, 64, A, None, 0, None), 2),
    ((A, 1, -1, 256, 64, A, A, A, 128, A, None, 0, None), 2),
    ((A, 1, 0, 256, 64, A, A, A, 128, A, None, 0, None), 0),     # M == 0: OK, nothing launched
    ((None, 1, 0, 256, 64, None, None, None, 128, None, None, 0, None), 0),
    ((None, 1, 1, 256, 64, A, A, A, 128, A, None, 0, None), 1),
    ((A, 1, 1, 256, 64, A, A, A, 128, B, None, 0, None), 3),
])
def test_gemm_w4a16_rejects(args, want):
    import bit_quantized_gemm_group_b200 as q
    assert q.lib().qg_gemm_w4a16(*args) == want


@pytest.mark.parametrize("fn,args,want", [
    ("qg_gemm_w8a8", (A, A, 4, 256, A, A, 72, A, None, None, 0, None), 2),     # N % 16
    ("qg_gemm_w8a8", (A, A, 4, 256, A, A, 64, A, B, None, 0, None), 3),        # misaligned debug output
    ("qg_gemm_w8a8", (A, None, 4, 256, A, A, 64, A, None, None, 0, None), 1),
    ("qg_gemm_w8a8", (None, None, 0, 256, None, None, 64, None, None, None, 0, None), 0),
    ("qg_gemm_w4a8", (A, A, 4, 256, A, A, 64, 64, A, None, None, 0, None), 2),  # group != 128
    ("qg_gemm_w4a8", (A, A, 4, 256, A, None, 64, 128, A, None, None, 0, None), 1),
    ("qg_smooth_quant_act_i8", (A, 4, 12, None, A, A, None), 2),                # K % 8
    ("qg_smooth_quant_act_i8", (A, 4, 16, B, A, A, None), 3),
    ("qg_smooth_quant_act_i8", (None, 0, 16, None, None, None, None), 0),
    ("qg_pack_nibbles", (A, 12, 16, A, None), 2),
    ("qg_pack_nibbles", (None, 16, 16, A, None), 1),
    ("qg_quantize_w8_channel", (A, None, 0, 16, A, A, None), 2),
    # outlier_split_w4(W, s, K, N, group, count, idx, codes8, s8, W_dense, stream)
    ("qg_outlier_split_w4", (A, None, 256, 64, 128, 9, A, A, A, A, None), 2),   # count above 8
    ("qg_outlier_split_w4", (A, None, 256, 64, 128, -1, A, A, A, A, None), 2),
    ("qg_outlier_split_w4", (A, None, 512, 64, 512, 3, A, A, A, A, None), 2),   # offsets must fit u8
    ("qg_outlier_split_w4", (A, None, 200, 64, 128, 3, A, A, A, A, None), 2),   # K % group
    ("qg_outlier_split_w4", (A, None, 256, 64, 128, 3, None, A, A, A, None), 1),
    ("qg_outlier_split_w4", (A, B, 256, 64, 128, 3, A, A, A, A, None), 3),
    # outlier_side_add(X, xdt, M, K, N, group, count, idx, codes8, s8, Y, stream)
    ("qg_outlier_side_add", (A, 7, 4, 256, 64, 128, 3, A, A, A, A, None), 4),
    ("qg_outlier_side_add", (A, 1, 4, 256, 64, 128, 3, A, A, None, A, None), 1),
    ("qg_outlier_side_add", (None, 1, 0, 256, 64, 128, 3, None, None, None, None, None), 0),
    ("qg_outlier_side_add", (A, 1, 4, 256, 64, 128, 3, A, A, A, B, None), 3),
    # gemm_w4a16_outlier: the side-path arguments are checked before the GEMM launches
    ("qg_gemm_w4a16_outlier", (A, 1, 4, 256, 64, A, A, A, 128, 9, A, A, A, A, None, 0, None), 2),
    ("qg_gemm_w4a16_outlier", (A, 1, 4, 256, 64, A, A, A, 128, 3, A, A, None, A, None, 0, None), 1),
    ("qg_gemm_w4a16_outlier", (A, 1, 4, 256, 60, A, A, A, 128, 3, A, A, A, A, None, 0, None), 2),   # GEMM's N % 8
    # gptq(Xcal, Mc, K, W, N, group, damp, codes, scales, zeros, ws, ws_bytes, stream)
    ("qg_gptq", (A, 16, 256, A, 64, 100, 0.01, A, A, A, A, 1 << 40, None), 2),    # group % 8
    ("qg_gptq", (A, 16, 200, A, 64, 128, 0.01, A, A, A, A, 1 << 40, None), 2),    # K % group
    ("qg_gptq", (A, 16, 256, A, 64, 128, 0.0, A, A, A, A, 1 << 40, None), 2),     # damp must be > 0
    ("qg_gptq", (A, 0, 256, A, 64, 128, 0.01, A, A, A, A, 1 << 40, None), 2),
    ("qg_gptq", (A, 16, 256, A, 64, 128, 0.01, A, A, A, None, 0, None), 1),       # workspace required
    ("qg_gptq", (A, 16, 256, A, 64, 128, 0.01, A, A, A, A, 1000, None), 10),      # too small
    ("qg_gptq", (A, 16, 256, A, 64, 128, 0.01, A, B, A, A, 1 << 40, None), 3),
    ("qg_prune24", (A, 48, 16, A, A, None), 2),                                # K % 32
    ("qg_prune24", (A, 64, 16, None, A, None), 1),
    ("qg_prune24", (A, 64, 16, A, B, None), 3),
    ("qg_pack24_vals", (A, A, 40, 16, A, None), 2),
    ("qg_pack24_vals", (A, None, 64, 16, A, None), 1),
    # gemm_w4a16_24(X, xdt, M, K, N, vals, meta, scales, zeros, group, Y, stream)
    ("qg_gemm_w4a16_24", (A, 9, 1, 256, 16, A, A, A, A, 128, A, None), 4),
    ("qg_gemm_w4a16_24", (A, 1, 1, 192, 16, A, A, A, A, 128, A, None), 2),   # K % 128
    ("qg_gemm_w4a16_24", (A, 1, 1, 256, 16, A, A, A, A, 64, A, None), 2),
    ("qg_gemm_w4a16_24", (None, 1, 0, 256, 16, None, None, None, None, 128, None, None), 0),
    ("qg_gemm_w4a16_24", (A, 1, 1, 256, 16, A, None, A, A, 128, A, None), 1),
    ("qg_gemm_w4a16_24", (A, 1, 1, 256, 16, A, A, A, A, 128, B, None), 3),
    # gptq_blocked(Xcal, Mc, K, W, N, group, damp, codes, scales, zeros, ws, ws_bytes, stream)
    ("qg_gptq_blocked", (A, 16, 256, A, 64, 100, 0.01, A, A, A, A, 1 << 40, None), 2),    # group % 8
    ("qg_gptq_blocked", (A, 16, 200, A, 64, 128, 0.01, A, A, A, A, 1 << 40, None), 2),    # K % group
    ("qg_gptq_blocked", (A, 16, 32768, A, 64, 128, 0.01, A, A, A, A, 1 << 40, None), 2),  # K > 16384
    ("qg_gptq_blocked", (A, 16, 256, A, 64, 128, 0.0, A, A, A, A, 1 << 40, None), 2),     # damp must be > 0
    ("qg_gptq_blocked", (A, 16, 256, A, 64, 128, 0.01, A, A, A, None, 0, None), 1),       # workspace required
    ("qg_gptq_blocked", (A, 16, 256, A, 64, 128, 0.01, A, A, A, A, 1000, None), 10),      # too small
    ("qg_gptq_blocked", (A, 16, 256, A, 64, 128, 0.01, A, B, A, A, 1 << 40, None), 3),
    # pack24_tc(vals, K, N, vals_tc, stream)
    ("qg_pack24_tc", (None, 256, 16, A, None), 1),
    ("qg_pack24_tc", (A, 200, 16, A, None), 2),                                # K % 128
    ("qg_pack24_tc", (A, 256, 16, A, None), 2),                                # not in place
    ("qg_pack24_tc", (A, 256, 16, B, None), 3),
    # gemm_w4a16_24_tc(X, xdt, M, K, N, vals_tc, meta, scales, zeros, group, Y, ws, ws_bytes, stream)
    ("qg_gemm_w4a16_24_tc", (A, 9, 1, 256, 32, A, A, A, A, 128, A, A, 1 << 30, None), 4),
    ("qg_gemm_w4a16_24_tc", (A, 1, 1, 256, 16, A, A, A, A, 128, A, A, 1 << 30, None), 2),   # N % 32
    ("qg_gemm_w4a16_24_tc", (A, 1, 1, 192, 32, A, A, A, A, 128, A, A, 1 << 30, None), 2),   # K % 128
    ("qg_gemm_w4a16_24_tc", (A, 1, 1, 256, 32, A, A, A, A, 64, A, A, 1 << 30, None), 2),    # group 128 only
    ("qg_gemm_w4a16_24_tc", (None, 1, 0, 256, 32, None, None, None, None, 128, None, None, 0, None), 0),
    ("qg_gemm_w4a16_24_tc", (A, 1, 1, 256, 32, A, A, A, A, 128, A, None, 0, None), 1),      # workspace required
    ("qg_gemm_w4a16_24_tc", (A, 1, 1, 256, 32, A, A, A, A, 128, B, A, 1 << 30, None), 3),
    ("qg_gemm_w4a16_24_tc", (A, 1, 1, 256, 32, A, A, A, A, 128, A, A, 100, None), 10),      # too small
    ("qg_awq_act_mean", (A, 0, 16, A, None), 2),
    ("qg_awq_act_mean", (None, 4, 16, A, None), 1),
    ("qg_awq_act_mean", (A, 4, 16, B, None), 3),
    ("qg_awq_scales", (A, 16, 1.5, A, A, None), 2),                            # alpha outside [0, 1]
    ("qg_awq_scales", (A, 16, -0.1, A, A, None), 2),
    ("qg_awq_scales", (A, 16, float("nan"), A, A, None), 2),
    ("qg_awq_scales", (A, 16, 0.5, None, A, None), 1),
    ("qg_awq_scale_act", (A, 4, 12, A, A, None), 2),                           # K % 8
    ("qg_awq_scale_act", (None, 0, 16, None, None, None), 0),
    ("qg_awq_scale_act", (A, 4, 16, B, A, None), 3),
    # awq_search(Xcal, Mc, K, W, N, group, n_grid, mse, best, s, inv_s, ws, ws_bytes, stream)
    ("qg_awq_search", (A, 4, 256, A, 64, 64, 5, A, A, A, A, A, 1 << 30, None), 2),   # group != 128
    ("qg_awq_search", (A, 4, 200, A, 64, 128, 5, A, A, A, A, A, 1 << 30, None), 2),  # K % 128
    ("qg_awq_search", (A, 4, 256, A, 60, 128, 5, A, A, A, A, A, 1 << 30, None), 2),  # N % 8
    ("qg_awq_search", (A, 4, 256, A, 64, 128, 0, A, A, A, A, A, 1 << 30, None), 2),  # empty grid
    ("qg_awq_search", (A, 0, 256, A, 64, 128, 5, A, A, A, A, A, 1 << 30, None), 2),  # no tokens
    ("qg_awq_search", (A, 4, 256, A, 64, 128, 5, A, A, A, A, None, 0, None), 1),     # workspace required
    ("qg_awq_search", (A, 4, 256, A, 64, 128, 5, A, A, A, A, A, 100, None), 10),     # workspace too small
    ("qg_awq_search", (A, 4, 256, A, 64, 128, 5, B, A, A, A, A, 1 << 30, None), 3),
])
def test_other_calls_reject(fn, args, want):
    import bit_quantized_gemm_group_b200 as q
    assert getattr(q.lib(), fn)(*args) == want


def test_smooth_scales_rejects_alpha():
    import bit_quantized_gemm_group_b200 as q
    f = q.lib().qg_smooth_scales
    assert f(A, 4, A, 16, 16, ctypes.c_float(1.5), A, A, None) == 2
    assert f(A, 4, A, 16, 16, ctypes.c_float(float("nan")), A, A, None) == 2


def test_workspace_size_and_too_small_workspace():
    import bit_quantized_gemm_group_b200 as q
    L = q.lib()
    need = L.qg_workspace_size(0, 32, 4096, 4096)
    assert need > 0
    assert L.qg_workspace_size(0, 1, 4096, 136) == 0       # N % 16 != 0: no workspace path
    assert L.qg_workspace_size(1, 16, 4096, 11008) > 0     # W8A8 below 128 tokens: stream-K partials
    assert L.qg_workspace_size(1, 128, 4096, 11008) == 0   # W8A8 tile kernel takes none
    assert L.qg_workspace_size(2, 17, 4096, 11008) > 0     # W4A8 at 17..127 tokens: stream-K partials
    assert L.qg_workspace_size(2, 16, 4096, 11008) == 0    # W4A8 at 16 tokens and fewer: split-K, none
    assert L.qg_workspace_size(2, 128, 4096, 11008) == 0   # W4A8 tile kernel takes none
    # the int8 stream-K kernels finish split slabs in the launch: one 64-bit publication
    # token per CTA (padded to 256 B), then one published NT x 128 tile of 4-byte sums per
    # CTA, NT the token tile (16 / 32 / 64 / 128); the plan has one CTA per SM (148 when
    # no GPU answers the query, as here or on a B200)
    tok = (148 * 8 + 255) // 256 * 256
    for M, nt in ((1, 16), (16, 16), (17, 32), (32, 32), (64, 64), (100, 128)):
        assert L.qg_workspace_size(1, M, 4096, 11008) == tok + 148 * nt * 128 * 4
    for M, nt in ((17, 32), (64, 64)):
        assert L.qg_workspace_size(2, M, 8192, 8192) == tok + 148 * nt * 128 * 4
    assert L.qg_workspace_size(0, 0, 4096, 4096) == 0
    # AWQ search: every buffer of one candidate, so at least codes + packed + outputs
    K, N, Mc = 4096, 12288, 512
    assert L.qg_workspace_size(3, Mc, K, N) >= K * N * 3 // 2 + Mc * N * 6 + Mc * K * 2
    assert L.qg_workspace_size(3, Mc, K, 12284) == 0
    # GPTQ: two K x K binary64 matrices and the binary64 weights, for any K a group divides
    assert L.qg_workspace_size(4, 16, 96, 5) >= 8 * (2 * 96 * 96 + 96 * 5)
    assert L.qg_workspace_size(4, 16, 100, 5) == 0
    assert L.qg_workspace_size(4, 16, 32768, 5) == 0
    # a workspace smaller than required is refused before any launch
    assert L.qg_gemm_w4a16(A, 1, 32, 4096, 4096, A, A, A, 128, A, A, need - 1, None) == 10
    assert L.qg_gemm_w4a16(A, 1, 32, 4096, 4096, A, A, A, 128, A, B, need, None) == 3
    need8 = L.qg_workspace_size(1, 16, 4096, 11008)
    assert L.qg_gemm_w8a8(A, A, 16, 4096, A, A, 11008, A, None, A, need8 - 1, None) == 10
    assert L.qg_gemm_w8a8(A, A, 16, 4096, A, A, 11008, A, None, B, need8, None) == 3
    need4 = L.qg_workspace_size(2, 32, 4096, 11008)
    assert L.qg_gemm_w4a8(A, A, 32, 4096, A, A, 11008, 128, A, None, A, need4 - 1, None) == 10
    assert L.qg_gemm_w4a8(A, A, 32, 4096, A, A, 11008, 128, A, None, B, need4, None) == 3


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="needs a host without a usable GPU: the call below launches with fake pointers")
def test_host_side_cuda_failure_is_reported():
    """A CUDA runtime failure on the host (here: no usable device) comes back as
    QG_ERR_CUDA with the failing call and the runtime's message, and the binding's
    exception carries that text."""
    import bit_quantized_gemm_group_b200 as q
    L = q.lib()
    assert L.qg_pack_nibbles(A, 16, 16, A, None) == q.QG_ERR_CUDA
    msg = L.qg_last_error().decode()
    assert "cudaGetLastError" in msg and len(msg) > len("cudaGetLastError(): ")
    assert L.qg_device_status(None) == q.QG_ERR_CUDA
    assert "cudaStreamSynchronize" in L.qg_last_error().decode()
    err = q.QgError(q.QG_ERR_CUDA, "qg_device_status")
    assert "QG_ERR_CUDA" in str(err) and "cudaStreamSynchronize" in str(err)
