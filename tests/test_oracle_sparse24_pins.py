"""Pins for the oracle's 2:4 structured sparsity + INT4 ("LLM inference cost: W8A8/W4A8
...", sec. 3.2): the 2 largest |w| of every 4 along K kept, the rest zero, then INT4
groups of 128; stored as the kept codes plus 4 bits of positions per 4-block.

Pins: a hand-derived column (tests/golden/hand_examples.json: the kept positions with
ties and the metadata word), numpy's stable sort as brute force for the selection, the
identity on weights that are already 2:4, the value packing (hand word and a round trip),
and the reference product against numpy's matmul of the dequantized sparse matrix.
They run on the CPU only.
"""
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        return json.load(f)["sparse24"]


def _kept(meta, K):
    """Kept positions [K/4][2][N] decoded from the metadata with numpy."""
    N = meta.shape[1]
    b = np.arange(K // 4)
    nib = (meta[b // 8] >> (4 * (b % 8))[:, None].astype(np.uint32)) & 0xF
    return np.stack([nib & 3, nib >> 2], axis=1).astype(np.int64).reshape(K // 4, 2, N)


def test_hand_column():
    h = _hand()[0]
    col = np.array(h["column_k0_to_k31"], np.float32)[:, None]
    Wp, meta = oracle.prune24(col)
    assert int(meta[0, 0]) == int(h["meta_word"], 16)
    kept = _kept(meta, 32)[:, :, 0]
    np.testing.assert_array_equal(kept, np.array(h["kept_positions_per_block"]))
    mask = np.zeros(32, bool)
    for bi, (a, c) in enumerate(h["kept_positions_per_block"]):
        mask[4 * bi + a] = mask[4 * bi + c] = True
    np.testing.assert_array_equal(Wp[:, 0], np.where(mask, col[:, 0], 0.0))


def test_selection_matches_a_stable_sort():
    rng = np.random.default_rng(1)
    K, N = 128, 24
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    W[8:12, 0] = [0.5, -0.5, 0.5, 0.1]           # ties on |w|
    W[20:24, 1] = 0.0                              # an all-zero block
    Wp, meta = oracle.prune24(W)
    kept = _kept(meta, K)
    for b in range(K // 4):
        blk = W[4 * b:4 * b + 4]
        for n in range(N):
            order = np.lexsort((np.arange(4), -np.abs(blk[:, n])))[:2]
            np.testing.assert_array_equal(kept[b, :, n], np.sort(order))
            keep = np.zeros(4, bool)
            keep[order] = True
            np.testing.assert_array_equal(Wp[4 * b:4 * b + 4, n], np.where(keep, blk[:, n], 0.0))


def test_identity_on_weights_already_two_of_four():
    rng = np.random.default_rng(2)
    K, N = 64, 10
    W = (rng.standard_normal((K, N)) + 3.0).astype(np.float32)  # no zeros
    for b in range(K // 4):
        for n in range(N):
            W[4 * b + rng.choice(4, 2, replace=False), n] = 0.0
    Wp, _ = oracle.prune24(W)
    np.testing.assert_array_equal(Wp, W)


def test_value_packing():
    h = _hand()[1]
    K = 32
    codes = np.zeros((K, 1), np.uint8)
    meta = np.zeros((1, 1), np.uint32)  # every block keeps positions 0 and 1
    for b in range(8):
        meta[0, 0] |= np.uint32(0x4) << np.uint32(4 * b)
    kv = h["kept_codes_in_k_order"]
    for j, c in enumerate(kv):  # kept value j sits at k = 4 (j // 2) + (j % 2)
        codes[4 * (j // 2) + (j % 2), 0] = c
    vals = oracle.pack24_vals(codes, meta)
    assert int(vals[0, 0]) == int(h["vals_word"], 16)
    # round trip on random codes and patterns
    rng = np.random.default_rng(3)
    K, N = 128, 8
    W = rng.standard_normal((K, N)).astype(np.float32)
    _, meta = oracle.prune24(W)
    codes = rng.integers(0, 16, (K, N)).astype(np.uint8)
    vals = oracle.pack24_vals(codes, meta)
    kept = _kept(meta, K)
    for kvi in range(K // 2):
        b, j = divmod(kvi, 2)
        got = (vals[kvi // 8] >> np.uint32(4 * (kvi % 8))) & 0xF
        np.testing.assert_array_equal(got, codes[4 * b + kept[b, j], np.arange(N)])


def test_reference_product_against_numpy():
    rng = np.random.default_rng(4)
    M, K, N = 5, 256, 20
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    Wp, meta = oracle.prune24(W)
    codes, scales, zeros, _ = oracle.quantize_w4_asym(Wp)
    vals = oracle.pack24_vals(codes, meta)
    y, b = oracle.gemm_w4a16_24_ref(X, vals, meta, scales, zeros)
    sc = oracle.f16_to_f32(scales).astype(np.float64)
    wd = (codes.astype(np.float64) - np.repeat(zeros.astype(np.float64), 128, 0)) * np.repeat(sc, 128, 0)
    mask = np.zeros((K, N), bool)
    kept = _kept(meta, K)
    for bi in range(K // 4):
        for j in range(2):
            mask[4 * bi + kept[bi, j], np.arange(N)] = True
    wd = np.where(mask, wd, 0.0)  # pruned positions are not stored: exactly 0
    np.testing.assert_allclose(y, X.astype(np.float64) @ wd, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(b, np.abs(X.astype(np.float64)) @ np.abs(wd), rtol=1e-12)
    assert mask.sum() == K * N // 2
