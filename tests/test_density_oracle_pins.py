"""Pins of the state density field oracle (oracle/density_oracle.cpp).

The oracle is held to things other than itself: two rows worked by hand
(tests/golden/density_field_tiny.txt); the closed form of a first-order sigma-delta
modulator (the ones among the first j cells number floor(U_j + 1/2), U_j the exact sum of
the targets of those cells), checked with exact rational arithmetic on inputs whose fp32
steps are exact; the error bounds that closed form implies (each value within 2 scale / len of
its input, and every prefix of the length-weighted errors within half a cell); exact values
at the row's extremes; the zero row; the cell partition; invariance under power-of-two
scaling. A dropped error feedback, a value given the wrong cells or a wrong sign in the
readout each fails one of them.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "density_field_tiny.txt")
K_MAMBA2 = 23             # K^2 = 529, about 4 d_state for d_state = 128
D_STATE = 128


def golden_rows():
    for ln in open(GOLDEN):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        name, s, scale, b, dec = [f.split() for f in ln.split("|")]
        yield name[0], np.array(s, np.float32), float(scale[0]), bytes(int(v, 16) for v in b), np.array(dec, float)


@pytest.mark.parametrize("row", list(golden_rows()), ids=lambda r: r[0])
def test_hand_worked_rows(row):
    _, s, scale, b, dec = row
    sc, bits = oracle.density_encode(s[None, :], 4)
    assert sc[0] == scale and bytes(bits[0]) == b
    np.testing.assert_array_equal(oracle.density_decode(sc, bits, 4, 4)[0], dec)


def cells_of(n, d, K):
    c = K * K
    return n * c // d, (n + 1) * c // d


def bit_list(bits_row, K):
    return [(int(bits_row[c >> 3]) >> (c & 7)) & 1 for c in range(K * K)]


def test_cell_partition():
    lens = [b - a for a, b in (cells_of(n, D_STATE, K_MAMBA2) for n in range(D_STATE))]
    assert sum(lens) == K_MAMBA2 ** 2 and set(lens) == {4, 5} and lens.count(5) == 529 - 4 * 128


def exact_rows(seed, rows, d):
    # v = k / 1024 exactly, scale a power of two: every fp32 step of the modulator is exact
    rng = np.random.default_rng(seed)
    k = rng.integers(-1024, 1025, (rows, d))
    k[:, rng.integers(0, d)] = 1024                   # the row's max |s| is the scale
    scale = 2.0 ** rng.integers(-6, 6, (rows, 1))
    return (k / 1024.0 * scale).astype(np.float32), k


@pytest.mark.parametrize("d,K", [(128, 23), (16, 8), (7, 3), (33, 12)])
def test_closed_form_of_the_modulator(d, K):
    s, k = exact_rows(d * 100 + K, 5, d)
    _, bits = oracle.density_encode(s, K)
    for r in range(s.shape[0]):
        got = bit_list(bits[r], K)
        U, ones = Fraction(0), 0
        for n in range(d):
            u = (Fraction(int(k[r, n]), 1024) + 1) / 2
            a, b = cells_of(n, d, K)
            for c in range(a, b):
                U += u
                ones += got[c]
                assert ones == (U + Fraction(1, 2)).__floor__(), (r, n, c)


def test_error_bounds_and_noise_shaping():
    rng = np.random.default_rng(7)
    s = (rng.standard_normal((64, D_STATE)) * rng.uniform(1e-3, 10, (64, 1))).astype(np.float32)
    scale, bits = oracle.density_encode(s, K_MAMBA2)
    dec = oracle.density_decode(scale, bits, D_STATE, K_MAMBA2)
    lens = np.array([b - a for a, b in (cells_of(n, D_STATE, K_MAMBA2) for n in range(D_STATE))], float)
    sc = scale.astype(np.float64)[:, None]
    err = dec - s.astype(np.float64)
    assert (np.abs(err) <= 2 * sc / lens[None, :] * (1 + 1e-6)).all()
    # first-order noise shaping: the length-weighted error of every prefix stays within half a cell
    prefix = np.cumsum(lens[None, :] * err / (2 * sc), axis=1)
    assert np.abs(prefix).max() <= 0.5 + 1e-5


def test_extremes_are_exact_and_scale_is_the_max():
    rng = np.random.default_rng(11)
    s = rng.standard_normal((16, D_STATE)).astype(np.float32)
    scale, bits = oracle.density_encode(s, K_MAMBA2)
    np.testing.assert_array_equal(scale, np.abs(s).max(axis=1))
    dec = oracle.density_decode(scale, bits, D_STATE, K_MAMBA2)
    at = np.abs(s) == scale[:, None]
    np.testing.assert_array_equal(dec[at], s[at].astype(np.float64))


def test_zero_row():
    scale, bits = oracle.density_encode(np.zeros((1, D_STATE), np.float32), K_MAMBA2)
    assert scale[0] == 0.0
    assert bit_list(bits[0], K_MAMBA2) == [1 - (c & 1) for c in range(K_MAMBA2 ** 2)]   # u = 1/2: 1 0 1 0 ...
    np.testing.assert_array_equal(oracle.density_decode(scale, bits, D_STATE, K_MAMBA2), 0.0)


def test_power_of_two_scaling():
    rng = np.random.default_rng(13)
    s = rng.standard_normal((8, D_STATE)).astype(np.float32)
    sc0, b0 = oracle.density_encode(s, K_MAMBA2)
    for p in (2.0 ** 7, 2.0 ** -9):
        sc, b = oracle.density_encode(s * np.float32(p), K_MAMBA2)
        np.testing.assert_array_equal(b, b0)
        np.testing.assert_array_equal(sc, sc0 * np.float32(p))
