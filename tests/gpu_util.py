"""Helpers shared by the GPU parity tests: move seeded inputs to the device, call the
library through its binding, bring results back as numpy arrays."""
import numpy as np
import torch

import bit_quantized_gemm_group_b200 as q


def cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def u16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def u32(t):
    return t.cpu().view(torch.int32).numpy().view(np.uint32)


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f16_to_f32(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float32)


def quant_w4_asym(W_np, s=None, group=128):
    """-> device (codes u8, scales int16 (fp16 bits), zeros u8, packed int32 (u32 bits))"""
    K, N = W_np.shape
    W = cuda(W_np)
    sd = None if s is None else cuda(s)
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    scales = torch.empty(K // group, N, dtype=torch.int16, device="cuda")
    zeros = torch.empty(K // group, N, dtype=torch.uint8, device="cuda")
    q.qg_quantize_w4_group(W, sd, group, False, codes, scales, zeros)
    packed = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    q.qg_pack_nibbles(codes, packed)
    return codes, scales, zeros, packed


def quant_w4_sym(W_np, s=None, group=128):
    K, N = W_np.shape
    W = cuda(W_np)
    sd = None if s is None else cuda(s)
    codes = torch.empty(K, N, dtype=torch.uint8, device="cuda")
    scales = torch.empty(K // group, N, dtype=torch.float32, device="cuda")
    q.qg_quantize_w4_group(W, sd, group, True, codes, scales, None)
    packed = torch.empty(K // 8, N, dtype=torch.int32, device="cuda")
    q.qg_pack_nibbles(codes, packed)
    return codes, scales, packed


def x_device(bits, dtype):
    return cuda(bits.view(np.int16), None).view(dtype)


def sample_rows(M, extra=4, seed=0):
    rows = {0, M - 1, M // 2}
    if M > 1:
        rows.add(1)
    if M > 64:
        rows.add(63)
    rng = np.random.default_rng(seed)
    rows.update(int(r) for r in rng.integers(0, M, extra))
    return np.array(sorted(rows), np.int64)
