"""Seeded synthetic inputs for the quantized linear layer.

Shared by the tests, the bench and the smoke check.  This module holds no step of
the method: it only draws the random tensors the workloads describe and rounds
activations to their storage dtype with torch's own conversions.  Both the CUDA
path and the CPU oracle receive the same arrays from here.

Workloads (shapes only; no model weights are involved):

* ``w4a16_tiny``    X [1x1024] fp16 ~N(0,1); W [1024x1024] ~N(0,0.02), 1% entries x8.
* ``w4a16_decode``  Llama-2-7B-shaped layers: M in {1,4,16,32};
                    (K,N) in {(4096,12288),(4096,4096),(4096,22016),(11008,4096)};
                    bf16 X ~N(0,1); W ~N(0,0.02), 1% entries x8.
* ``w8a8``          X [M x 4096] bf16 ~N(0,1) with 8 fixed channels x50, M in {16,256,2048};
                    W [4096 x 11008] ~N(0,0.02); smoothing alpha = 0.5.
* ``w4a16_prefill`` 70B-shaped MLP: M in {4096,8192}; (K,N) in {(8192,28672),(28672,8192)};
                    bf16 X ~N(0,1); W ~N(0,0.015), 0.5% entries x8.
* ``w4a8``          X [M x 8192] bf16 ~N(0,1) with 16 fixed channels x30, M in {1,64,1024};
                    W [8192 x 8192] ~N(0,0.02); smoothing alpha = 0.5.
* ``awq``           AWQ scale search for the decode layers' INT4 weights: calibration X
                    [512 x 4096] bf16 ~N(0,1) with 8 fixed channels x50; W [4096 x 12288]
                    ~N(0,0.02), 1% entries x8 (the decode weights); 21 grid points.

Exact-arithmetic operands (``exact_*``): quantized operands drawn directly -- INT4 codes,
zero points, power-of-two scales and small integer activations -- on which every
product and partial sum of the GEMMs is exact in binary32 (the bounds are stated per
function), so any correct kernel returns the exact product rounded once.

Random streams: every draw comes from ``numpy.random.Generator(PCG64)`` seeded by
``SeedSequence([seed, stream, *shape])`` with one stream id per tensor role, so a
tensor does not change when another one is added.  The outlier channels of X are a
seeded sample without replacement of K, shared by X and its calibration batch.
"""
from __future__ import annotations

import numpy as np
import torch

S_W, S_X, S_XCAL, S_MASK, S_CHANNELS, S_EXACT = 1, 2, 3, 4, 5, 6

CONFIGS = {
    "w4a16_tiny": dict(M=[1], KN=[(1024, 1024)], xdtype="f16", w_std=0.02,
                       outlier_frac=0.01, outlier_mult=8.0, group=128),
    "w4a16_decode": dict(M=[1, 4, 16, 32], KN=[(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)],
                         xdtype="bf16", w_std=0.02, outlier_frac=0.01, outlier_mult=8.0, group=128),
    "w8a8": dict(M=[16, 256, 2048], KN=[(4096, 11008)], xdtype="bf16", w_std=0.02,
                 x_channels=8, x_mult=50.0, alpha=0.5, calib_tokens=512),
    "w4a16_prefill": dict(M=[4096, 8192], KN=[(8192, 28672), (28672, 8192)], xdtype="bf16", w_std=0.015,
                          outlier_frac=0.005, outlier_mult=8.0, group=128),
    "w4a8": dict(M=[1, 64, 1024], KN=[(8192, 8192)], xdtype="bf16", w_std=0.02,
                 x_channels=16, x_mult=30.0, alpha=0.5, calib_tokens=512, group=128),
    "awq": dict(M=[512], KN=[(4096, 12288)], xdtype="bf16", w_std=0.02, outlier_frac=0.01, outlier_mult=8.0,
                x_channels=8, x_mult=50.0, calib_tokens=512, n_grid=21, group=128),
}


def rng(seed: int, stream: int, *shape: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, *shape])))


def weights(K: int, N: int, std: float, outlier_frac: float = 0.0, outlier_mult: float = 1.0,
            seed: int = 0) -> np.ndarray:
    """W [K][N] fp32 ~ N(0, std) with an independent Bernoulli(outlier_frac) mask scaled by outlier_mult."""
    W = rng(seed, S_W, K, N).standard_normal((K, N), dtype=np.float32)
    W *= np.float32(std)
    if outlier_frac > 0.0:
        mask = rng(seed, S_MASK, K, N).random((K, N), dtype=np.float32) < np.float32(outlier_frac)
        W[mask] *= np.float32(outlier_mult)
    return W


def outlier_channels(K: int, count: int, seed: int = 0) -> np.ndarray:
    if count <= 0:
        return np.zeros(0, np.int64)
    return np.sort(rng(seed, S_CHANNELS, K, count).choice(K, size=count, replace=False)).astype(np.int64)


def activations(M: int, K: int, dtype: str = "bf16", channels: int = 0, mult: float = 1.0,
                seed: int = 0, stream: int = S_X):
    """X [M][K] ~ N(0,1), `channels` fixed channels scaled by `mult`, rounded to bf16/fp16.

    Returns (values as fp32 -- exactly representable in `dtype`, raw 16-bit patterns)."""
    X = rng(seed, stream, M, K).standard_normal((M, K), dtype=np.float32)
    ch = outlier_channels(K, channels, seed)
    if ch.size:
        X[:, ch] *= np.float32(mult)
    t = torch.from_numpy(X)
    t16 = t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float16)
    bits = t16.view(torch.int16).numpy().view(np.uint16).copy()
    vals = t16.to(torch.float32).numpy().copy()
    return vals, bits


def calibration(K: int, cfg: dict, seed: int = 0):
    """A separate calibration batch drawn like the workload's X (same outlier channels)."""
    return activations(cfg["calib_tokens"], K, cfg["xdtype"], cfg.get("x_channels", 0),
                       cfg.get("x_mult", 1.0), seed, stream=S_XCAL)


def workload_weights(name: str, K: int, N: int, seed: int = 0) -> np.ndarray:
    cfg = CONFIGS[name]
    return weights(K, N, cfg["w_std"], cfg.get("outlier_frac", 0.0), cfg.get("outlier_mult", 1.0), seed)


def workload_activations(name: str, M: int, K: int, seed: int = 0):
    cfg = CONFIGS[name]
    return activations(M, K, cfg["xdtype"], cfg.get("x_channels", 0), cfg.get("x_mult", 1.0), seed)


# ---------------------------------------------------------------------------
# exact-arithmetic operands
# ---------------------------------------------------------------------------
def exact_w4_asym(K: int, N: int, group: int = 128, e_min: int = -2, seed: int = 0):
    """Asymmetric INT4 operands drawn directly: codes u8 in [0, 15], zero points u8 in
    [0, 15], scales 2^e with e in [e_min, 0] as fp16 bit patterns [K/group][N].
    Every (q - z) * 2^e is exact in bf16 and fp16."""
    r = rng(seed, S_EXACT, 1, K, N)
    codes = r.integers(0, 16, (K, N)).astype(np.uint8)
    zeros = r.integers(0, 16, (K // group, N)).astype(np.uint8)
    e = r.integers(e_min, 1, (K // group, N))
    scales = np.asarray(2.0 ** e, np.float16).view(np.uint16).copy()
    return codes, scales, zeros


def exact_w4_sym(K: int, N: int, group: int = 128, e_min: int = -2, seed: int = 0):
    """Symmetric INT4 operands drawn directly: codes int8 in [-7, 7], fp32 scales 2^e
    with e in [e_min, 0], [K/group][N]."""
    r = rng(seed, S_EXACT, 2, K, N)
    codes = r.integers(-7, 8, (K, N)).astype(np.int8)
    e = r.integers(e_min, 1, (K // group, N))
    return codes, (2.0 ** e).astype(np.float32)


def exact_activations(M: int, K: int, xmax: int = 8, dtype: str = "bf16", seed: int = 0):
    """Integer activations in [-xmax, xmax] (exact in bf16 and fp16).
    Returns (values as fp32, raw 16-bit patterns) like ``activations``."""
    X = rng(seed, S_EXACT, 3, M, K).integers(-xmax, xmax + 1, (M, K)).astype(np.float32)
    t = torch.from_numpy(X)
    t16 = t.to(torch.bfloat16) if dtype == "bf16" else t.to(torch.float16)
    return X, t16.view(torch.int16).numpy().view(np.uint16).copy()


def exact_act_i8(M: int, K: int, qmax: int = 31, seed: int = 0):
    """INT8 activation codes in [-qmax, qmax] with power-of-two token scales 2^f,
    f in [-9, -6]."""
    r = rng(seed, S_EXACT, 4, M, K)
    Xq = r.integers(-qmax, qmax + 1, (M, K)).astype(np.int8)
    t = (2.0 ** r.integers(-9, -5, M)).astype(np.float32)
    return Xq, t
