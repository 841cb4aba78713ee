"""The synthetic workloads follow their stated recipe (CPU only).

The five workloads stand in for the pages' trained layers: seeded draws with
the shapes, outlier densities and outlier structures of the configurations
(uniform, global top-|w|, 2% of rows and columns, Zipf(1.2) per-row counts).
These tests pin the generator to that recipe, so a change to it shows up
here rather than as a silent change of what the kernels are measured on.
"""
import numpy as np
import pytest

import synth

# round-half-up(density * rows * cols) of each workload
NNZ = {"c0": 10486, "c1": 75497, "c2": 450888, "c3": 225444, "c4_q": 443023}

_cache = {}


def cfg(name):
    if name not in _cache:
        _cache[name] = synth.make_config(name, batch=1)
    return _cache[name]


def f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


@pytest.mark.parametrize("name", sorted(NNZ))
def test_shape_nnz_and_csr_form(name):
    p = cfg(name)
    assert p.nnz == NNZ[name]
    rp = np.asarray(p.row_ptr)
    assert rp[0] == 0 and rp[-1] == p.nnz and np.all(np.diff(rp) >= 0)
    ci = np.asarray(p.col_idx)
    assert ci.min() >= 0 and ci.max() < p.cols
    # columns strictly increasing inside every row
    inc = np.diff(ci) > 0
    row_start = np.zeros(p.nnz, dtype=bool)
    row_start[rp[:-1][rp[:-1] < p.nnz]] = True
    assert np.all(inc | row_start[1:])
    assert np.all(np.isfinite(f16(p.values)))
    assert p.codes.shape == (p.rows, p.cols) and int(p.codes.max()) < (1 << p.bits)


def test_generation_is_deterministic():
    a, b = synth.make_config("c0", batch=1), synth.make_config("c0", batch=1)
    for f in ("codes", "table", "row_ptr", "col_idx", "values", "x"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_c0_outliers_are_the_largest_weights():
    """Global top-|w|: every outlier is at least as large as any table entry,
    since the tables are quantiles of the weights left in the dense part."""
    p = cfg("c0")
    assert np.abs(f16(p.values)).min() >= np.abs(f16(p.table)).max() * (1 - 2.0 ** -10)


def test_c2_outliers_concentrate_in_2pct_of_rows_and_columns():
    """A quarter of the outliers lies in 2% of the rows, a quarter in 2% of
    the columns (plus those rows' and columns' share of the uniform half)."""
    p = cfg("c2")
    rows = np.sort(np.diff(p.row_ptr))[::-1]
    cols = np.sort(np.bincount(p.col_idx, minlength=p.cols))[::-1]
    n_r, n_c = int(np.ceil(0.02 * p.rows)), int(np.ceil(0.02 * p.cols))
    assert (n_r, n_c) == (221, 82)
    assert rows[:n_r].sum() >= p.nnz // 4
    assert cols[:n_c].sum() >= p.nnz // 4
    # and the rest is spread: the median row holds about the uniform share
    assert 0.5 * 0.005 * p.cols <= np.median(rows) <= 2.0 * 0.005 * p.cols


def test_c3_zipf_counts():
    """Rank-based Zipf(1.2) counts clipped at the row width: four rows are
    entirely outliers; the tail of the distribution is heavy (p99 ~ 744)."""
    p = cfg("c3")
    counts = np.diff(p.row_ptr)
    assert int((counts == p.cols).sum()) == 4
    assert 700 <= np.percentile(counts, 99) <= 790
    assert int((counts > 50).sum()) == pytest.approx(398, abs=20)
    # count of rank r is proportional to r^-1.2 for the unclipped ranks
    s = np.sort(counts)[::-1].astype(np.float64)
    ratio = s[9] / s[99]
    assert ratio == pytest.approx(10.0 ** 1.2, rel=0.05)


def test_affine_groups_are_well_formed():
    p = cfg("c2")
    scales, zeros = f16(p.table), f16(p.zeros)
    assert p.table.shape == (p.rows, p.cols // 16) == p.zeros.shape
    assert np.all(scales > 0)
    assert np.all(zeros == np.round(zeros)) and zeros.min() >= 0 and zeros.max() <= 7


def test_activations_are_standard_normal_fp16():
    p = cfg("c2")
    x = f16(p.x[0])
    assert abs(x.mean()) < 0.1 and 0.9 < x.std() < 1.1
