"""Pins of the oracle's decomposition step (outlier selection, CSR build and
the two quantizers) against what the pages and independent routines fix,
with planted mistakes that each fail at least one pin.  Host only."""
import json
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def spiky(rng, rows, cols, frac=0.01):
    """fp32 weights: N(0, 0.02^2) plus Laplace(0, 0.2) spikes, as the workloads."""
    w = rng.normal(0.0, 0.02, (rows, cols))
    n = int(frac * rows * cols)
    pos = rng.choice(rows * cols, n, replace=False)
    w.reshape(-1)[pos] += rng.laplace(0.0, 0.2, n)
    return w.astype(np.float32)


def holes_of(w, nnz):
    """The nnz largest |w| (ties: the lower row-major index first), by numpy's stable sort."""
    order = np.argsort(-np.abs(w.astype(np.float64)).reshape(-1), kind="stable")
    hole = np.zeros(w.size, bool)
    hole[order[:nnz]] = True
    return hole.reshape(w.shape)


def pin_golden_affine(orc):
    g = json.load(open(os.path.join(GOLDEN, "decompose_example.json")))
    w = np.array(g["w"], np.float32).reshape(g["rows"], g["cols"])
    codes, table, zeros, rp, ci, va = orc.decompose(w, g["bits"], "affine", g["nnz"])
    assert list(rp) == g["row_ptr"] and list(ci) == g["col_idx"]
    assert [hex(int(v)) for v in va] == g["values"]
    assert hex(int(table[0, 0])) == g["scale"] and hex(int(zeros[0, 0])) == g["zero"]
    assert list(codes[0]) == g["codes"]


def pin_topk_and_csr(orc):
    """Outliers are the nnz largest |w| by numpy's stable sort, ties (equal
    |w| of either sign, planted) taken in row-major order; the CSR lists them
    row by row, columns ascending, values rounded to fp16."""
    rng = np.random.default_rng(3)
    w = spiky(rng, 23, 80)
    w[5, 7], w[2, 9], w[5, 60], w[11, 0] = 0.75, -0.75, 0.75, -0.75   # a tie straddling the cut
    nnz = int(np.sum(np.abs(w) > 0.75)) + 2
    _, _, _, rp, ci, va = orc.decompose(w, 3, "lut", nnz)
    hole = holes_of(w, nnz)
    r, c = np.nonzero(hole)
    assert np.array_equal(rp, np.concatenate([[0], np.cumsum(hole.sum(axis=1))]))
    assert np.array_equal(ci, c)
    assert np.array_equal(va, w[r, c].astype(np.float16).view(np.uint16))
    assert hole[2, 9] and hole[5, 7] and not hole[5, 60] and not hole[11, 0]


def pin_affine_matches_generator(orc):
    """The affine quantizer equals the numpy generator's (scale from the
    widened range, fp16 rounding, rint, clipping) on spiky fp32 weights."""
    rng = np.random.default_rng(4)
    for bits in (3, 4):
        w = spiky(rng, 17, 96)
        w[4] = np.abs(w[4]) + 0.1              # all-positive groups: the range must widen to 0
        w[9] = -np.abs(w[9]) - 0.05            # all-negative groups
        # range 6e-7: scale = fp16(6e-7 / (2^b - 1)) rounds down to a coarse
        # subnormal, -min / scale passes 2^b - 1 and the zero must be clipped
        w[12] = np.tile(np.linspace(-6e-7, -1e-8, 16), 6)
        nnz = int(0.01 * w.size)
        codes, table, zeros, *_ = orc.decompose(w, bits, "affine", nnz)
        wd = np.where(holes_of(w, nnz), 0.0, w.astype(np.float64))
        c2, s2, z2 = synth._quantize_affine(wd, bits)
        assert np.array_equal(codes, c2) and np.array_equal(table, s2) and np.array_equal(zeros, z2)
    # a group of zeros only (scale would be 0): scale 1, zero 0, codes 0
    w = np.zeros((1, 16), np.float32)
    codes, table, zeros, *_ = orc.decompose(w, 3, "affine", 0)
    assert table[0, 0] == 0x3C00 and zeros[0, 0] == 0 and np.all(codes == 0)


def pin_lut_quantiles(orc):
    """Table centroids are numpy.quantile's linear quantiles at (2k+1)/2^(b+1)
    of the row's dense weights; on multiples of 1/64 every interpolation is
    exact, so the two agree bit for bit; codes are the nearest centroid with
    ties to the lower index, as the numpy generator's; a row made only of
    outliers gets zero centroids."""
    rng = np.random.default_rng(5)
    for bits in (3, 4):
        K = 1 << bits
        w = (rng.integers(-64, 65, (9, 64)) / 64.0).astype(np.float32)
        w[3] = 10.0 + np.arange(64)          # row 3: all outliers
        nnz = 64 + 5
        codes, table, _, *_ = orc.decompose(w, bits, "lut", nnz)
        hole = holes_of(w, nnz)
        assert hole[3].all()
        levels = (2.0 * np.arange(K) + 1.0) / (2.0 * K)
        for i in range(9):
            vals = w[i][~hole[i]].astype(np.float64)
            want = np.quantile(vals, levels) if vals.size else np.zeros(K)
            assert np.array_equal(table[i], want.astype(np.float16).view(np.uint16)), i
        c2, t2 = synth._quantize_lut(np.where(hole, 0.0, w.astype(np.float64)), hole, bits)
        assert np.array_equal(codes, c2) and np.array_equal(table, t2)


PINS = [pin_golden_affine, pin_topk_and_csr, pin_affine_matches_generator, pin_lut_quantiles]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


MUTANTS = {
    "ties_by_higher_index": ("return a->i < b->i ? -1 : (a->i > b->i ? 1 : 0);",
                             "return a->i > b->i ? -1 : (a->i < b->i ? 1 : 0);"),
    "smallest_first": ("return a->a > b->a ? -1 : 1;", "return a->a < b->a ? -1 : 1;"),
    "range_not_widened": ("double mn = 0.0, mx = 0.0, sv, z;", "double mn = 1e300, mx = -1e300, sv, z;"),
    "holes_keep_weight": ("double v = hole[t] ? 0.0 : (double)w[t];\n                    if (v < mn)",
                          "double v = (double)w[t];\n                    if (v < mn)"),
    "zero_not_clipped": ("z = z < 0.0 ? 0.0 : (z > qmax ? qmax : z);", "z = z;"),
    "scale_levels_8": ("s16 = oracle_double_to_half((mx - mn) / qmax);", "s16 = oracle_double_to_half((mx - mn) / K);"),
    "quantile_levels": ("double p = (2.0 * q + 1.0) / (2.0 * K);", "double p = (double)q / (double)K;"),
    "nearest_ties_upper": ("if (fabs(v - cent[q]) < bd) {", "if (fabs(v - cent[q]) <= bd) {"),
    "outlier_not_removed": ("hole[it[t].i] = 1;", "hole[it[t].i] = 0;"),
    "csr_value_rounding": ("values[k] = oracle_double_to_half((double)w[i * cols + j]);",
                           "values[k] = oracle_double_to_half((double)(float)(w[i * cols + j] * 1.0009765625f));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    old, new = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, name
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        path = os.path.join(tmp, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        mutant = oracle.load(path, os.path.join(tmp, "mutant.so"))
        failed = []
        for pin in PINS:
            try:
                pin(mutant)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"planted mistake {name} passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
