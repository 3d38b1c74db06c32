"""The fp64 oracle against its pins (CPU only), and mutants of it against the same pins."""
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

import oracle as oracle_pkg
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(oracle, pin):
    assert pin(oracle) is None


def test_truncated_power_general_degree(oracle):
    # The FlashKAN abstract states the bounded-coordinate form for degree k;
    # the oracle's recursion is written for any degree.
    assert pins.pin_truncated_power(oracle, grids=((8, -1.0, 1.0), (5, -3.0, 3.0)), degrees=(1, 2, 4, 5)) is None


@pytest.mark.parametrize("k", [1, 2, 4, 5])
def test_general_degree_pins(oracle, k):
    # Spline degree k (the FlashKAN abstract: "k sequential passes for degree-k splines", normalised
    # coordinate clamped to [0, k+1]): partition of unity, non-negativity and k+1 non-zeros,
    # degree-k polynomial reproduction through forward and dx, and finite differences.
    assert pins.pin_partition_of_unity(oracle, k=k) is None
    assert pins.pin_nonneg_local(oracle, k=k) is None
    assert pins.pin_marsden(oracle, k=k) is None
    assert pins.pin_finite_difference(oracle, k=k) is None


def test_golden_rows_sum(oracle):
    # the fixture itself: weights sum to 1, derivatives to 0 (exact rationals)
    for row in pins.read_golden():
        assert sum(row[1:5]) == 1
        assert sum(row[5:9]) == 0


def test_backward_skips(oracle):
    rng = np.random.default_rng(3)
    x = rng.uniform(-1, 1, (9, 3)); coef = rng.normal(size=(2, 3, 11)); dY = rng.normal(size=(9, 2))
    dx, dcoef, dwb = oracle.backward(x, coef, dY, 8, -1.0, 1.0, want_dcoef=False)
    assert dcoef is None and dwb is None and dx.shape == (9, 3)
    dx2, dcoef2, _ = oracle.backward(x, coef, dY, 8, -1.0, 1.0, want_dx=False)
    assert dx2 is None and dcoef2.shape == coef.shape


def test_thread_count_invariance(oracle):
    rng = np.random.default_rng(4)
    x = rng.uniform(-1.2, 1.2, (101, 7)); coef = rng.normal(size=(5, 7, 11)); dY = rng.normal(size=(101, 5))
    wb = rng.normal(size=(5, 7))
    y1 = oracle.forward(x, coef, 8, -1.0, 1.0, w_base=wb, nthreads=1)
    y8 = oracle.forward(x, coef, 8, -1.0, 1.0, w_base=wb, nthreads=8)
    assert np.array_equal(y1, y8)
    g1 = oracle.backward(x, coef, dY, 8, -1.0, 1.0, w_base=wb, nthreads=1)
    g3 = oracle.backward(x, coef, dY, 8, -1.0, 1.0, w_base=wb, nthreads=3)
    assert np.array_equal(g1[0], g3[0])
    np.testing.assert_allclose(g1[1], g3[1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(g1[2], g3[2], rtol=0, atol=1e-13)


def test_empty_batch(oracle):
    x = np.zeros((0, 3)); coef = np.ones((2, 3, 11)); dY = np.zeros((0, 2))
    assert oracle.forward(x, coef, 8, -1.0, 1.0).shape == (0, 2)
    dx, dcoef, _ = oracle.backward(x, coef, dY, 8, -1.0, 1.0)
    assert dx.shape == (0, 3) and np.all(dcoef == 0)


# --------------------------------------------------------------------------
# Mutation check: each plausible mistake, planted in a private copy of the
# oracle source on the CPU, must make at least one pin fail.
MUTANTS = {
    "closed_degree0_interval": ("x < t[j + 1]) ? 1.0", "x <= t[j + 1]) ? 1.0"),
    "derivative_sign": ("dB[j] = a * prev[j] - c * prev[j + 1];", "dB[j] = a * prev[j] + c * prev[j + 1];"),
    "dropped_right_term": ("cur[j] = left + right;", "cur[j] = left;"),
    "knot_offset": ("(double)(j - k) * (hi - lo)", "(double)(j - k + 1) * (hi - lo)"),
    "forward_coef_index": ("acc += cj[i * nb + m] * bv;", "acc += cj[m * J->in + i] * bv;"),
    "forward_base_transposed": ("acc += J->w_base[j * J->in + i] * Srow[i];",
                                "acc += J->w_base[i * J->out + j] * Srow[i];"),
    "dx_drops_base": ("if (J->w_base) d += J->w_base[j * J->in + i] * dSrow[i];", ""),
    "dsilu_sign": ("return s * (1.0 + x * (1.0 - s));", "return s * (1.0 + x * (1.0 + s));"),
    "dcoef_uses_derivative": ("double bv = Brow[i * nb + m];\n                        if (bv != 0.0) pj[i * nb + m] += bv * g;",
                              "double bv = dBrow[i * nb + m];\n                        if (bv != 0.0) pj[i * nb + m] += bv * g;"),
    "dx_wrong_dY_index": ("acc += dy[j] * d;", "acc += dy[0] * d;"),
    "dwb_uses_dsilu": ("J->dwb_part[j * J->in + i] += Srow[i] * dy[j];", "J->dwb_part[j * J->in + i] += dSrow[i] * dy[j];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(oracle_pkg._SRC).read()
    before, after = MUTANTS[name]
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = src.replace(before, after)
    csrc = tmp_path / "kan_oracle_mutant.c"
    csrc.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", str(csrc), "-o", str(so), "-lm"],
                   check=True)
    mutant = oracle_pkg.Oracle(oracle_pkg.load(str(so)))
    fails = pins.run_all(mutant)
    assert fails, f"mutant {name} passed every pin"
