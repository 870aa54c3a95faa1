"""Pins of the block-frame oracle (residual add + RMS norm, oracle/block_oracle.cpp).

The oracle is held to things other than itself: two cases worked by hand from the
definition (tests/golden/block_rmsnorm.txt), the norm's invariants (unit mean square with
w = 1 and eps = 0, invariance under exact scaling, odd symmetry), the fp32 residual as
IEEE single-precision addition (numpy float32), per-token independence and the all-zero
row. A dropped eps, a sum in place of the mean, a misplaced weight index or a wrong sign
each fails one of them.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_rmsnorm.txt")


def golden_cases():
    for ln in open(GOLDEN):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        head, r, delta, w, r_new, factor, out = [f.split() for f in ln.split("|")]
        name, d, eps = head[0], int(head[1]), float(head[2])
        dl = None if delta == ["-"] else np.array([int(v, 16) for v in delta], np.uint16)[None, :]
        yield name, d, eps, np.array(r, np.float32)[None, :], dl, np.array(w, np.float32), \
            np.array(r_new, np.float32), float(factor[0]), np.array(out, np.float64)


@pytest.mark.parametrize("case", list(golden_cases()), ids=lambda c: c[0])
def test_hand_worked_cases(case):
    name, d, eps, r, dl, w, r_new, factor, out = case
    got = oracle.add_rmsnorm(r, dl, w, eps)
    np.testing.assert_array_equal(got["resid"][0], r_new)
    assert got["r"][0] == pytest.approx(factor, rel=1e-15)
    np.testing.assert_allclose(got["out"][0], out, rtol=1e-15, atol=1e-300)


def rand(seed, m, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((m, d)) * rng.uniform(0.1, 10, (m, 1))).astype(np.float32)


def test_unit_mean_square_with_unit_weights_and_no_eps():
    r = rand(1, 5, 2048)
    got = oracle.add_rmsnorm(r, None, np.ones(2048, np.float32), 0.0)
    np.testing.assert_allclose(np.mean(got["out"] ** 2, axis=1), 1.0, rtol=1e-13)


def test_invariant_under_exact_scaling_and_odd():
    r = rand(2, 3, 512)
    w = np.random.default_rng(3).uniform(0.5, 1.5, 512).astype(np.float32)
    base = oracle.add_rmsnorm(r, None, w, 0.0)["out"]
    for k in (2.0 ** 5, 2.0 ** -7):
        np.testing.assert_allclose(oracle.add_rmsnorm(r * np.float32(k), None, w, 0.0)["out"], base, rtol=1e-14)
    np.testing.assert_array_equal(oracle.add_rmsnorm(-r, None, w, 0.0)["out"], -base)


def test_weights_scale_each_channel():
    r = rand(4, 2, 256)
    w = np.random.default_rng(5).uniform(0.5, 1.5, 256).astype(np.float32)
    ones = oracle.add_rmsnorm(r, None, np.ones(256, np.float32), 1e-5)["out"]
    got = oracle.add_rmsnorm(r, None, w, 1e-5)["out"]
    np.testing.assert_allclose(got, ones * w.astype(np.float64)[None, :], rtol=1e-15)


def test_residual_is_ieee_single_addition():
    m, d = 4, 1024
    r = rand(6, m, d)
    df = rand(7, m, d)
    db = (df.view(np.uint32) >> 16).astype(np.uint16)        # bf16 bits (truncated values)
    dbf = (db.astype(np.uint32) << 16).view(np.float32)
    np.testing.assert_array_equal(oracle.add_rmsnorm(r, df, np.ones(d, np.float32), 1e-5)["resid"], r + df)
    np.testing.assert_array_equal(oracle.add_rmsnorm(r, db, np.ones(d, np.float32), 1e-5)["resid"], r + dbf)
    np.testing.assert_array_equal(oracle.add_rmsnorm(r, None, np.ones(d, np.float32), 1e-5)["resid"], r)


def test_tokens_are_independent():
    r = rand(8, 6, 384)
    w = np.random.default_rng(9).uniform(0.5, 1.5, 384).astype(np.float32)
    all_ = oracle.add_rmsnorm(r, None, w, 1e-5)
    for t in range(6):
        one = oracle.add_rmsnorm(r[t:t + 1], None, w, 1e-5)
        np.testing.assert_array_equal(one["out"][0], all_["out"][t])


def test_zero_row_gives_zeros_and_the_eps_factor():
    got = oracle.add_rmsnorm(np.zeros((1, 64), np.float32), None, np.ones(64, np.float32), 0.25)
    np.testing.assert_array_equal(got["out"], 0.0)
    assert got["r"][0] == 2.0
