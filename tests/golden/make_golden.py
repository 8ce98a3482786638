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
    out = dict(codes=codes, scales=scales, zeros=zeros, packed=packed, y=y, b=b, s=s, inv=inv, xq=xq, t=t,
               qs=qs, ss=ss)
    # the rows added after the hot path: AWQ, the INT8 outlier side path, 2:4, GPTQ
    Xb, _ = synth.activations(16, K, "bf16", channels=4, mult=50.0, seed=1)
    mse, best, s_a, inv_a, st = oracle.awq_search(Xb, W, n_grid=5)
    assert st == 0
    out.update(awq_mse=mse, awq_best=np.array([best]), awq_s=s_a, awq_inv=inv_a)
    idx, c8, s8, dense, st = oracle.outlier_split(W)
    assert st == 0
    out.update(out_idx=idx, out_c8=c8, out_s8=s8, out_dense=dense)
    Wp, meta = oracle.prune24(W)
    c24, sc24, z24, _ = oracle.quantize_w4_asym(Wp)
    vals = oracle.pack24_vals(c24, meta)
    y24, _ = oracle.gemm_w4a16_24_ref(X, vals, meta, sc24, z24)
    out.update(sp_meta=meta, sp_vals=vals, sp_y=y24)
    gc, gs, gz, st = oracle.gptq(Xb, W)
    assert st == 0
    out.update(gptq_codes=gc, gptq_scales=gs, gptq_zeros=gz)
    return out


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regress.npz")
    np.savez_compressed(out, **make())
    print("wrote", out)
