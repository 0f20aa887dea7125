"""Pins for the oracle's Hadamard rotation and index quantisers.

'Token 的一生：DSV4 架构与 DSpark' §4: index queries and keys are rotated by a
Hadamard transform before FP8/FP4 quantisation (§3.1).  Pins: the Sylvester
matrix against its closed form (-1)^popcount(i&j), scipy's construction and
H H^T = nI; exact invariance of dot products under the normalised rotation;
quantisers that reproduce exactly-representable inputs bit for bit and stay
within the formats' half-step error bounds.
"""
import json
import os

import numpy as np
import scipy.linalg

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_hadamard_closed_form_and_library(orc):
    for n in [1, 2, 4, 8, 16, 32, 64, 128]:
        h = orc.hadamard_matrix(n).astype(np.int64)
        i = np.arange(n)[:, None]
        j = np.arange(n)[None, :]
        closed = np.where(np.vectorize(lambda a: bin(a).count("1") % 2)(i & j) == 0, 1, -1)
        assert np.array_equal(h, closed)
        assert np.array_equal(h, scipy.linalg.hadamard(n))
        assert np.array_equal(h @ h.T, n * np.eye(n, dtype=np.int64))


def test_hadamard_golden(orc):
    with open(os.path.join(GOLD, "hadamard_h4.json")) as f:
        g = json.load(f)
    assert orc.hadamard_matrix(2).tolist() == g["H2"]
    assert orc.hadamard_matrix(4).tolist() == g["H4"]


def test_rotation_preserves_dot_products(orc):
    rng = np.random.default_rng(0)
    for n in [64, 128]:
        x = rng.standard_normal((50, n))
        y = rng.standard_normal((50, n))
        rx, ry = orc.hadamard_rotate(x), orc.hadamard_rotate(y)
        assert np.allclose((rx * ry).sum(1), (x * y).sum(1), rtol=1e-12, atol=1e-12)
        # unnormalised: (Hx).(Hy) = n x.y
        assert np.allclose((rx * ry).sum(1) * n, (x * y).sum(1) * n, rtol=1e-12)
        # the normalised transform is a symmetric orthogonal involution
        assert np.allclose(orc.hadamard_rotate(rx), x, atol=1e-12)
        e0 = np.zeros(n)
        e0[0] = 1
        assert np.allclose(orc.hadamard_rotate(e0[None]), 1 / np.sqrt(n))


def test_fp8_rows_exact_inputs_round_trip(orc):
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 0x7F, size=(40, 128)).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=codes.shape) * 0x80).astype(np.uint8)
    codes[:, 5] = 0x7E                        # every row holds the max code
    s = 2.0 ** rng.integers(-8, 4, size=40)
    table = orc.e4m3_table()
    x = table[codes] * s[:, None]
    c2, s2 = orc.quant_fp8_rows(x)
    assert np.array_equal(s2, s.astype(np.float32))
    # -0 codes come back as -0: compare values and sign bits
    assert np.array_equal(c2, codes)


def test_fp8_rows_error_bound_and_zero_row(orc):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((200, 128)) * np.exp(rng.standard_normal((200, 1)))
    x[3] = 0.0
    codes, s = orc.quant_fp8_rows(x)
    deq = orc.dequant_fp8_rows(codes, s)
    assert s[3] == 1.0 and (codes[3] & 0x7F == 0).all()
    amax = np.abs(x).max(1)
    # half a step of E4M3 around v is <= 2^-4 |v| for normals, 2^-10 s for subnormals
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s[:, None].astype(np.float64)) * (1 + 1e-6)
    assert (np.abs(deq - x) <= bound + 1e-30).all()
    big = np.argmax(np.abs(x), axis=1)
    nz = amax > 0
    assert ((codes[np.arange(200), big] & 0x7F)[nz] == 0x7E).all()


def test_fp4_rows_exact_inputs_round_trip(orc):
    """Values built as e2m1 * ue4m3 * s_t with a full-scale element in every
    block and a 448 block scale somewhere come back bit for bit."""
    rng = np.random.default_rng(3)
    rows, n = 30, 128
    st = 2.0 ** -5
    sb = rng.integers(0x08, 0x7F, size=(rows, n // 16)).astype(np.uint8)
    sb[:, 2] = 0x7E
    codes = rng.integers(0, 16, size=(rows, n)).astype(np.uint8)
    codes[:, ::16] = 7 | (rng.integers(0, 2, size=(rows, n // 16)) * 8).astype(np.uint8)
    e2 = orc.e2m1_table()
    ue = orc.e4m3_table()
    x = e2[codes] * ue[np.repeat(sb, 16, axis=1)] * st
    c2, b2, s2 = orc.quant_fp4_rows(x)
    assert np.array_equal(s2, np.full(rows, st, dtype=np.float32))
    assert np.array_equal(b2, sb)
    # a -0 input code 8 comes back as 8 (sign kept)
    assert np.array_equal(c2, codes)


def test_fp4_rows_error_bound(orc):
    rng = np.random.default_rng(4)
    x = rng.standard_t(3, size=(100, 64))
    codes, bsc, rsc = orc.quant_fp4_rows(x)
    deq = orc.dequant_fp4_rows(codes, bsc, rsc)
    # half a step of E2M1 is at most 1 (between 4 and 6) in units of sb*s_t,
    # and the block max lands within one rounding of 6 units
    unit = orc.e4m3_table()[np.repeat(bsc, 16, axis=1)] * rsc[:, None]
    assert (np.abs(deq - x) <= 1.0 * unit * (1 + 1e-6) + 1e-30).all()
    # relative error of the block scale itself is at most 2^-4 (E4M3 half step)
    ab = np.abs(x).reshape(100, 4, 16).max(2)
    sbv = ab / (6 * rsc[:, None].astype(np.float64))
    sbq = orc.e4m3_table()[bsc]
    ok = sbv > 2.0 ** -6
    assert (np.abs(sbq - sbv)[ok] <= sbv[ok] * 2.0 ** -4 * (1 + 1e-5)).all()


def test_pack_fp4_nibble_order(orc):
    c = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    p = orc.pack_fp4(c)
    assert p.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(orc.unpack_fp4(p), c)
