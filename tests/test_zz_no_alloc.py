"""The allocation-free W4A16 entry point (qg_gemm_w4a16_noalloc), called through the C ABI.

It serves callers that cannot allocate device memory where they run the GEMM: code
being captured into a CUDA graph (no allocation inside a capture), operators inside a
host framework that owns every device allocation and hands the operator no allocator,
and latency-bound paths where an allocation's implicit synchronisation is not
acceptable.  Its scratch is a static device array instead of a caller workspace.

The entry point runs the same kernels with the same launch plan as the workspace
entry point, so its output must be bit-identical to that call's; it is also checked
against the oracle.  Shapes run from the largest launch to the smallest and every
second call uses different activations, so partial tiles left in the shared array
by an earlier call would show up.  This file is collected last on purpose: if it
fails, a run that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bf16_to_f32, quant_w4_asym, u16, x_device

pytestmark = pytest.mark.gpu

# largest scratch need first, then smaller ones (one process, one static array)
SHAPES = [(4096, 12288, 32), (11008, 4096, 8), (4096, 4096, 1), (1024, 1024, 3)]


def test_noalloc_matches_workspace_entry_point_and_oracle():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_quantized_gemm_group_b200 as q
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for K, N, M in SHAPES:
        W = synth.workload_weights("w4a16_decode", K, N)
        codes, scales, zeros, packed = quant_w4_asym(W)
        c_o, s_o, z_o, _ = oracle.quantize_w4_asym(W)
        p_o = oracle.pack_nibbles(c_o)
        ws = torch.zeros(q.qg_workspace_size(q.QG_OP_GEMM_W4A16, M, K, N), dtype=torch.uint8, device="cuda")
        for call in range(2):   # two calls in a row share the static array
            X, Xb = synth.activations(M, K, "bf16", seed=100 * call + M)
            Xd = x_device(Xb, torch.bfloat16)
            Y_ws = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            q.qg_gemm_w4a16(Xd, packed, scales, zeros, Y_ws, workspace=ws)
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            st = q.lib().qg_gemm_w4a16_noalloc(ctypes.c_void_p(Xd.data_ptr()), q.QG_BF16, M, K, N,
                                               ctypes.c_void_p(packed.data_ptr()),
                                               ctypes.c_void_p(scales.data_ptr()),
                                               ctypes.c_void_p(zeros.data_ptr()), 128,
                                               ctypes.c_void_p(Y.data_ptr()), stream)
            assert st == q.QG_OK, q.qg_status_string(st)
            assert q.qg_device_status() == q.QG_OK
            assert torch.equal(Y.view(torch.int16), Y_ws.view(torch.int16)), f"K={K} N={N} M={M} call {call}"
            yref, b = oracle.gemm_w4a16_ref(X, p_o, s_o, z_o)
            y = bf16_to_f32(u16(Y))
            assert oracle.within_tolerance(y, yref, b).all(), f"K={K} N={N} M={M} call {call}"

