"""Write oracle_regress.npz: the oracle's outputs on one seeded tiny case.

Calls only oracle/ (and the seeded input generator).  Re-run it only when a change to the
oracle's arithmetic is justified by a passage of the pages; name that passage in the commit.
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def make():
    K, N, M = 256, 64, 3
    W = synth.weights(K, N, 0.02, 0.01, 8.0, seed=0)
    X, xbits = synth.activations(M, K, "f16", seed=0)
    codes, scales, zeros, st = oracle.quantize_w4_asym(W)
    assert st == 0
    packed = oracle.pack_nibbles(codes)
    y, b = oracle.gemm_w4a16_ref(X, packed, scales, zeros)
    Xc, _ = synth.activations(32, K, "bf16", channels=4, mult=50.0, seed=0, stream=synth.S_XCAL)
    s, inv, _ = oracle.smooth_scales(Xc, W, 0.5)
    Xa, _ = synth.activations(M, K, "bf16", channels=4, mult=50.0, seed=0)
    xq, t, _ = oracle.smooth_quant_act_i8(Xa, inv)
    qs, ss, _ = oracle.quantize_w4_sym(W, s_smooth=s)
    return dict(codes=codes, scales=scales, zeros=zeros, packed=packed, y=y, b=b, s=s, inv=inv, xq=xq, t=t,
                qs=qs, ss=ss)


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regress.npz")
    np.savez_compressed(out, **make())
    print("wrote", out)
