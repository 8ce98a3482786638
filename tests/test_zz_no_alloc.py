"""The allocation-free W4A16 entry point (qg_gemm_w4a16_noalloc), called through the C ABI.

It serves callers that cannot allocate device memory where they run the GEMM (inside
a graph capture, inside a framework that owns the allocator, on latency-bound paths),
so its scratch is a static device array instead of a workspace.  This file is
collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_f32, quant_w4_asym, u16, x_device

pytestmark = pytest.mark.gpu

SHAPES = [(4096, 4096, 1), (4096, 12288, 32), (11008, 4096, 8), (1024, 1024, 3)]


@pytest.mark.parametrize("K,N,M", SHAPES)
def test_noalloc_matches_workspace_entry_point_twice(K, N, M):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_quantized_gemm_group_b200 as q
    W = synth.workload_weights("w4a16_decode", K, N)
    codes, scales, zeros, packed = quant_w4_asym(W)
    X, Xb = synth.activations(M, K, "bf16", seed=7 + M)
    Xd = x_device(Xb, torch.bfloat16)
    # the existing entry point, with a workspace of its own
    ws = torch.zeros(q.qg_workspace_size(q.QG_OP_GEMM_W4A16, M, K, N), dtype=torch.uint8, device="cuda")
    Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    q.qg_gemm_w4a16(Xd, packed, scales, zeros, Y_ref, workspace=ws)
    assert q.qg_device_status() == q.QG_OK
    c_o, s_o, z_o, _ = oracle.quantize_w4_asym(W)
    _, b = oracle.gemm_w4a16_ref(X, oracle.pack_nibbles(c_o), s_o, z_o)
    y_ref = bf16_to_f32(u16(Y_ref))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):   # two calls in a row share the static scratch
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = q.lib().qg_gemm_w4a16_noalloc(ctypes.c_void_p(Xd.data_ptr()), q.QG_BF16, M, K, N,
                                           ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                           ctypes.c_void_p(zeros.data_ptr()), 128, ctypes.c_void_p(Y.data_ptr()),
                                           stream)
        assert st == q.QG_OK, q.qg_status_string(st)
        assert q.qg_device_status() == q.QG_OK
        y = bf16_to_f32(u16(Y))
        assert (np.abs(y - y_ref) <= 1e-2 * b + 1e-3).all(), f"call {call}"
