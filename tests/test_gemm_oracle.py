"""Pins of the oracle's fused-GEMM functions (oracle/__init__.py, section
"decode fused into the consuming GEMM"), each against something other than
the oracle itself: hand-derived tile positions, a pure-Python triple loop,
closed forms of the product and known BF16 values.  No GPU."""
import os
import struct

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gemm_tile.txt")


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


def test_tile_positions_match_hand_derivation():
    rows = [tuple(int(v) for v in line.split()) for line in open(GOLDEN)
            if line.strip() and not line.startswith("#")]
    assert len(rows) == 14
    for k, n, pos, value in rows:
        w = np.arange(k * n, dtype=np.uint16)
        assert int(oracle.gemm_tile(w, k, n)[pos]) == value, (k, n, pos)


@pytest.mark.parametrize("k,n", [(64, 128), (128, 384), (320, 256)])
def test_untile_inverts_tile(k, n):
    w = np.random.default_rng(k + n).integers(0, 1 << 16, k * n, dtype=np.uint16)
    t = oracle.gemm_tile(w, k, n)
    assert sorted(t.tolist()) == sorted(w.tolist())  # a permutation
    assert np.array_equal(oracle.gemm_untile(t, k, n).reshape(-1), w)
    # every tile is one contiguous 8192-weight run of 128 output rows x 64 inputs
    tiles = t.reshape(-1, 128, 64)
    W = w.reshape(k, n)
    nb, kb = 1 % (n // 128), (k // 64) - 1
    assert np.array_equal(tiles[nb * (k // 64) + kb], W[64 * kb: 64 * kb + 64, 128 * nb: 128 * nb + 128].T)


def _bf16(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0] >> 16  # exact for values with 8 significant bits


def test_bf16_values():
    got = oracle.bf16_to_float(np.array([0x3F80, 0xC000, 0x0001, 0x7F7F, 0x8000], np.uint16))
    assert got[0] == 1.0 and got[1] == -2.0 and got[2] == 2.0 ** -133 and got[4] == 0.0
    assert got[3] == (2 - 2 ** -7) * 2.0 ** 127


def test_product_equals_triple_loop():
    g = np.random.default_rng(7)
    m, k, n = 2, 64, 128
    xs = [float(v) for v in g.integers(-8, 9, m * k) / 8]
    ws = [float(v) for v in g.integers(-16, 17, k * n) / 32]
    xb = np.array([_bf16(v) for v in xs], np.uint16)
    wb = np.array([_bf16(v) for v in ws], np.uint16)
    y = oracle.gemm(xb, wb, m, k, n)
    for i in range(m):
        for j in range(0, n, 17):
            want = sum(xs[i * k + q] * ws[q * n + j] for q in range(k))
            assert y[i, j] == want, (i, j)
    assert np.array_equal(oracle.gemm_abs(xb, wb, m, k, n), np.abs(oracle.bf16_to_float(xb).reshape(m, k))
                          @ np.abs(oracle.bf16_to_float(wb).reshape(k, n)))


def test_one_hot_rows_select_weight_rows():
    """x row i = e_{k_i}: y row i is row k_i of W exactly (catches a transposed operand)."""
    k, n = 128, 256
    w = np.random.default_rng(3).integers(0, 0x3F00, k * n, dtype=np.uint16)
    picks = [0, 5, 64, 127]
    x = np.zeros((len(picks), k), np.uint16)
    for i, p in enumerate(picks):
        x[i, p] = 0x3F80  # 1.0
    y = oracle.gemm(x.reshape(-1), w, len(picks), k, n)
    W = oracle.bf16_to_float(w).reshape(k, n)
    for i, p in enumerate(picks):
        assert np.array_equal(y[i], W[p])


def test_decode_gemm_of_a_tiled_container():
    """Compress the tiled weights, then decode_gemm = the product with the
    original (untiled) weights."""
    k, n, m = 128, 256, 3
    g = np.random.default_rng(11)
    w = (np.asarray(g.standard_normal(k * n) * 0.02, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    x = (np.asarray(g.standard_normal(m * k), np.float32).view(np.uint32) >> 16).astype(np.uint16)
    c = oracle.compress(oracle.gemm_tile(w, k, n), "bf16", tile_threads=32)
    assert np.array_equal(oracle.decode_gemm(c, x, m, k, n), oracle.gemm(x, w, m, k, n))
