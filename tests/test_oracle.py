"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Every check below is written as a ``pin_*`` function of an oracle instance so
that ``test_planted_mistakes_are_caught`` can run the same checks against
copies of oracle.c with one mistake planted in each (a dropped term, a wrong
sign, a wrong index, a transposed operand, a wrong rounding rule) and show
that every planted mistake fails at least one pin.
"""
import json
import os
import shutil
import tempfile
import types
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def problem(rows, cols, bits, mode, codes, table, zeros, row_ptr, col_idx, values, x):
    return types.SimpleNamespace(
        rows=rows, cols=cols, bits=bits, mode=mode,
        codes=np.asarray(codes, np.uint8).reshape(rows, cols),
        table=np.asarray(table, np.uint16),
        zeros=None if zeros is None else np.asarray(zeros, np.uint16),
        row_ptr=np.asarray(row_ptr, np.int32), col_idx=np.asarray(col_idx, np.int32),
        values=np.asarray(values, np.uint16),
        x=np.asarray(x, np.uint16).reshape(-1, cols))


def np_h2d(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def np_d2h(v):
    with np.errstate(over="ignore"):
        return np.asarray(v, np.float64).astype(np.float16).view(np.uint16)


def random_finite_f16(rng, shape, lo_exp=-24, hi_exp=15):
    """fp16 bit patterns spread over many binades (subnormals included)."""
    e = rng.integers(lo_exp, hi_exp + 1, size=shape).astype(np.float64)
    v = rng.uniform(1.0, 2.0, size=shape) * np.exp2(e) * rng.choice([-1.0, 1.0], size=shape)
    h = np_d2h(v)
    h = np.where((h & 0x7C00) == 0x7C00, np.uint16(0x3C00), h)
    return h.astype(np.uint16)


def random_problem(rng, rows, cols, bits, mode, batch, nnz_per_row_max=4,
                   scale_exp=(-6, 2)):
    K = 1 << bits
    codes = rng.integers(0, K, size=(rows, cols))
    if mode == "lut":
        table = random_finite_f16(rng, (rows, K), -20, 4)
        zeros = None
    elif mode == "bitplane":
        table = random_finite_f16(rng, (rows, cols // (32 << bits), bits + 1), -12, 2)
        zeros = None
    else:
        table = random_finite_f16(rng, (rows, cols // 16), *scale_exp)
        zeros = np_d2h(rng.integers(0, K, size=(rows, cols // 16)))
    counts = rng.integers(0, nnz_per_row_max + 1, size=rows)
    row_ptr = np.concatenate([[0], np.cumsum(counts)])
    col_idx = np.concatenate([np.sort(rng.choice(cols, c, replace=False)) for c in counts]
                             + [np.zeros(0, np.int64)])
    values = random_finite_f16(rng, (int(row_ptr[-1]),), -10, 3)
    x = random_finite_f16(rng, (batch, cols), -12, 3)
    return problem(rows, cols, bits, mode, codes, table, zeros, row_ptr, col_idx, values, x)


# ------------------------------------------------------------------ fp16 pins

def pin_half_to_double_exhaustive(orc):
    """Every binary16 pattern decodes to numpy's value (NaNs stay NaN)."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.half_to_double(h)
    want = np_h2d(h)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def pin_double_to_half(orc):
    """Round trip of every finite pattern; every tie between neighbours (both
    signs) and its two closest doubles; overflow edges; 10^6 random doubles
    over all binades - all against numpy's own fp64 -> fp16 rounding."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (h & 0x7C00) != 0x7C00
    hf = h[finite]
    assert np.array_equal(orc.double_to_half(np_h2d(hf)), hf)
    pos = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo, hi = np_h2d(pos), np_h2d(pos + 1)
    mid = (lo + hi) / 2.0            # exact in fp64
    probes = np.concatenate([mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)])
    probes = np.concatenate([probes, -probes,
                             [65504.0, 65519.999, 65520.0, 65536.0, 1e300, -1e300,
                              2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -26, 1e-300,
                              -0.0, 0.0, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25]])
    rng = np.random.default_rng(7)
    rnd = rng.uniform(1, 2, 10 ** 6) * np.exp2(rng.integers(-30, 17, 10 ** 6)) \
        * rng.choice([-1.0, 1.0], 10 ** 6)
    for v in (probes, rnd):
        assert np.array_equal(orc.double_to_half(v), np_d2h(v))


# ------------------------------------------------------------------ format pins

def pin_csr_example(orc):
    """The SpQR CSR example rebuilds the page's matrix, exactly, when the dense
    part is all zero: as a 4x7 and as an 8x8 matrix, in table mode, and in
    affine mode with every code equal to its group's zero (holes decode to 0)."""
    g = json.load(open(os.path.join(GOLDEN, "csr_example.json")))
    vals = [int(v, 16) for v in g["values_f16_bits"]]
    assert list(np_h2d(vals)) == g["values_real"]
    want = np.array(g["dense_4x7"], dtype=np.float64)
    p = problem(4, 7, 3, "lut", np.zeros(28), np.zeros((4, 8)), None,
                g["row_ptr_4x7"], g["col_idx"], vals, np.zeros(7))
    got = orc.materialize(p)
    assert np.array_equal(got, want)
    p8 = problem(8, 8, 3, "lut", np.zeros(64), np.zeros((8, 8)), None,
                 g["row_ptr_8x8"], g["col_idx"], vals, np.zeros(8))
    want8 = np.zeros((8, 8))
    want8[:4, :7] = want
    assert np.array_equal(orc.materialize(p8), want8)
    pa = problem(4, 16, 3, "affine", np.full(64, 3), np.full((4, 1), 0x3C00),
                 np.full((4, 1), 0x4200), g["row_ptr_4x7"], g["col_idx"], vals,
                 np.zeros(16))
    wa = np.zeros((4, 16))
    wa[:, :7] = want
    assert np.array_equal(orc.materialize(pa), wa)


def pin_lut_decode_identity(orc):
    """Decoding codes 0..2^b-1 of a row returns that row's table, bit for bit
    (two rows with different tables, both code widths)."""
    rng = np.random.default_rng(11)
    for bits in (3, 4):
        K = 1 << bits
        table = random_finite_f16(rng, (2, K))
        codes = np.tile(np.arange(K), (2, 2))
        p = problem(2, 2 * K, bits, "lut", codes, table, None, [0, 0, 0], [], [],
                    np.zeros(2 * K))
        wd = orc.decode(p)
        assert np.array_equal(wd[:, :K], table) and np.array_equal(wd[:, K:], table)


def pin_affine_decode_golden(orc):
    """Hand-worked scale*(q-zero) values, ties and subnormals included."""
    g = json.load(open(os.path.join(GOLDEN, "affine_decode.json")))
    for c in g["cases"]:
        p = problem(1, 16, 3, "affine", np.full(16, c["q"]), [[int(c["scale"], 16)]],
                    [[int(c["zero"], 16)]], [0, 0], [], [], np.zeros(16))
        got = orc.decode(p)
        assert np.all(got == int(c["expect"], 16)), (c, hex(int(got[0, 0])))


def pin_affine_group_layout(orc):
    """Columns 0..15 use group 0, 16..31 group 1; each row its own groups."""
    codes = np.tile(np.arange(32) % 8, (2, 1))
    scales = np_d2h([[1.0, 2.0], [4.0, 0.5]])
    zeros = np_d2h([[0.0, 1.0], [2.0, 0.0]])
    p = problem(2, 32, 3, "affine", codes, scales, zeros, [0, 0, 0], [], [], np.zeros(32))
    q = np.arange(32) % 8
    want = np.stack([np.where(np.arange(32) < 16, 1.0 * q, 2.0 * (q - 1)),
                     np.where(np.arange(32) < 16, 4.0 * (q - 2), 0.5 * q)])
    assert np.array_equal(np_h2d(orc.decode(p)), want)


def bp_group(k):
    """Inputs per coefficient group of a bit-plane matrix with k planes."""
    return 32 << k


def pin_bitplane_decode_golden(orc):
    """Hand-worked C0 + sum_i C_i b_i values (BPDQ page, "Formulation de la
    Grille Variable"): plane order, ties, subnormals, overflow, and one
    rounding of the exact sum rather than one per addition."""
    g = json.load(open(os.path.join(GOLDEN, "bitplane_decode.json")))
    for c in g["cases"]:
        k = c["k"]
        K, G = 1 << k, bp_group(k)
        codes = np.tile(np.arange(K), G // K)
        coef = [[[int(v, 16) for v in c["coef"]]]]
        p = problem(1, G, k, "bitplane", codes, coef, None, [0, 0], [], [], np.zeros(G))
        got = orc.decode(p)[0]
        want = np.array([int(v, 16) for v in c["expect"]], np.uint16)
        assert np.array_equal(got, np.tile(want, G // K)), (c["why"], [hex(int(v)) for v in got[:K]])


def pin_bitplane_group_layout(orc):
    """Group g of row r covers columns g*32*2^k .. (g+1)*32*2^k - 1 and has
    its own coefficients; with C0 = 10 r + g, C1 = 1, C2 = 2 (, C3 = 4) the
    weight is the integer C0 + q."""
    for k in (2, 3):
        G, K = bp_group(k), 1 << k
        cols = 2 * G
        codes = np.tile(np.arange(cols) % K, (2, 1))
        coef = np.zeros((2, 2, k + 1))
        for r in range(2):
            for g in range(2):
                coef[r, g] = [10 * r + g] + [2.0 ** i for i in range(k)]
        p = problem(2, cols, k, "bitplane", codes, np_d2h(coef), None, [0, 0, 0], [], [], np.zeros(cols))
        grp = np.arange(cols) // G
        want = np.stack([10 * r + grp + np.arange(cols) % K for r in range(2)]).astype(np.float64)
        assert np.array_equal(np_h2d(orc.decode(p)), want)


def pin_bitplane_uniform_grid_is_affine(orc):
    """A bit-plane group with C_i = s * 2^(i-1) and C0 = -s * z is the
    uniform grid s * (q - z): it decodes exactly as the (separately pinned)
    affine decode with scale s and zero z, for every code."""
    rng = np.random.default_rng(21)
    for k in (2, 3):
        G, K = bp_group(k), 1 << k
        for _ in range(20):
            m = int(rng.integers(1, 128))              # <= 7 significant bits: s * z stays exact
            e = int(rng.integers(-20, 4))
            s = m * 2.0 ** e
            z = int(rng.integers(0, K))
            coef = [[np_d2h([0.0 - s * z] + [s * 2.0 ** i for i in range(k)])]]   # +0 when z = 0
            codes = np.tile(np.arange(K), G // K)
            bp = problem(1, G, k, "bitplane", codes, coef, None, [0, 0], [], [], np.zeros(G))
            af = problem(1, G, 3, "affine", codes, np.full((1, G // 16), np_d2h(s)),
                         np.full((1, G // 16), np_d2h(float(z))), [0, 0], [], [], np.zeros(G))
            assert np.array_equal(orc.decode(bp), orc.decode(af)), (k, s, z)


def pin_intgrid_decode_golden(orc):
    """Hand-worked fp16(scale * q) on the unconstrained integer grid (the
    Huffman-coded PTQ reading): large |q|, ties, subnormal scales."""
    g = json.load(open(os.path.join(GOLDEN, "intgrid_decode.json")))
    for c in g["cases"]:
        q = np.zeros(16, np.int16)
        q[:len(c["q"])] = c["q"]
        p = problem(1, 16, 14, "intgrid", np.zeros(16), [[int(c["scale"], 16)]], None, [0, 0], [], [],
                    np.zeros(16))
        p.codes = q.reshape(1, 16)
        got = orc.decode(p)[0, :len(c["q"])]
        assert [hex(int(v)) for v in got] == [hex(int(v, 16)) for v in c["expect"]], c["why"]


def pin_intgrid_group_layout(orc):
    """Columns 16g .. 16g+15 of row r use scale [r][g]; with q in 0..7 and
    power-of-two scales the weights are exact."""
    q = np.tile(np.arange(48) % 8, (2, 1)).astype(np.int16)
    scales = np_d2h([[1.0, 2.0, 0.5], [4.0, 0.25, 8.0]])
    p = problem(2, 48, 14, "intgrid", np.zeros(96), scales, None, [0, 0, 0], [], [], np.zeros(48))
    p.codes = q
    want = q * np.repeat(np_h2d(scales), 16, axis=1)
    assert np.array_equal(np_h2d(orc.decode(p)), want)


def pin_two_axis_golden(orc):
    """The hand-worked two-axis example (SINQ page, "Mise a l'echelle sur deux
    axes"): What = r_i c_j Wd_ij plus the unscaled outliers, and its product."""
    g = json.load(open(os.path.join(GOLDEN, "two_axis_example.json")))
    h = lambda v: [int(t, 16) for t in v]  # noqa: E731
    p = problem(g["rows"], g["cols"], g["bits"], "lut", np.array(g["codes"]).reshape(-1),
                [h(r) for r in g["table"]], None, g["row_ptr"], g["col_idx"], h(g["values"]), h(g["x"]))
    p.row_scale = np.array(h(g["row_scale"]), np.uint16)
    p.col_scale = np.array(h(g["col_scale"]), np.uint16)
    assert np.array_equal(orc.materialize(p), np.array(g["what"]))
    y, bd = orc.gemv(p)
    assert np.array_equal(y[0], np.array(g["y"])) and np.array_equal(bd[0], np.array(g["bound"]))


def pin_two_axis_unit_scales(orc):
    """All-one row and column scales leave every result of the plain product
    unchanged, bit for bit (every mode)."""
    rng = np.random.default_rng(31)
    for bits, mode, cols in ((3, "lut", 48), (4, "affine", 64), (2, "bitplane", 256)):
        p = random_problem(rng, 6, cols, bits, mode, 2)
        y0, b0 = orc.gemv(p)
        w0 = orc.materialize(p)
        p.row_scale = np.full(p.rows, 0x3C00, np.uint16)
        p.col_scale = np.full(p.cols, 0x3C00, np.uint16)
        y1, b1 = orc.gemv(p)
        assert np.array_equal(y0, y1) and np.array_equal(b0, b1)
        assert np.array_equal(w0, orc.materialize(p))


# ------------------------------------------------------------------ product pins

def exact_reference(p):
    """y and bound in exact rational arithmetic: decode each weight through
    fractions (affine: one rounding to fp16 via numpy), add outliers, sum."""
    K = 1 << p.bits
    W = [[None] * p.cols for _ in range(p.rows)]
    for i in range(p.rows):
        for j in range(p.cols):
            q = int(p.codes[i, j])
            if p.mode == "lut":
                W[i][j] = Fraction(float(np_h2d(p.table[i, q])))
            elif p.mode == "bitplane":
                G = 32 << p.bits
                c = [Fraction(float(v)) for v in np_h2d(p.table[i, j // G])]
                exact = c[0] + sum(c[t] for t in range(1, p.bits + 1) if (q >> (t - 1)) & 1)
                W[i][j] = Fraction(float(np_h2d(np_d2h(float(exact)))))
            else:
                s = Fraction(float(np_h2d(p.table[i, j // 16])))
                z = Fraction(float(np_h2d(p.zeros[i, j // 16])))
                W[i][j] = Fraction(float(np_h2d(np_d2h(float(s * (q - z))))))
        for k in range(int(p.row_ptr[i]), int(p.row_ptr[i + 1])):
            W[i][int(p.col_idx[k])] += Fraction(float(np_h2d(p.values[k])))
    xs = [[Fraction(float(v)) for v in np_h2d(row)] for row in p.x]
    y = [[sum(W[i][j] * xs[b][j] for j in range(p.cols)) for i in range(p.rows)]
         for b in range(len(xs))]
    bd = [[sum(abs(W[i][j]) * abs(xs[b][j]) for j in range(p.cols)) for i in range(p.rows)]
          for b in range(len(xs))]
    return y, bd


def pin_gemv_exact(orc):
    """y_ref and bound equal the exact rational result within fp64's own
    summation bound (n+2) * 2^-52 * bound, on small random problems of both
    modes and code widths, several rows, a batch of 3 and scattered outliers."""
    rng = np.random.default_rng(5)
    for bits, mode, cols in ((3, "lut", 32), (4, "lut", 32), (3, "affine", 32), (4, "affine", 32),
                             (2, "bitplane", 256), (3, "bitplane", 256)):
        p = random_problem(rng, 5, cols, bits, mode, 3)
        y, bd = orc.gemv(p)
        ye, be = exact_reference(p)
        tol = (p.cols + 2) * 2.0 ** -52
        for b in range(3):
            for i in range(p.rows):
                be_f = float(be[b][i])
                assert abs(y[b, i] - float(ye[b][i])) <= tol * be_f + 1e-300, (bits, mode, b, i)
                assert abs(bd[b, i] - be_f) <= tol * be_f + 1e-300, (bits, mode, b, i)


def pin_special_cases(orc):
    """x = 0 gives y = 0 and bound = 0 exactly; a one-hot x on an outlier-free
    column returns that column of W_dense exactly; an empty CSR is the dense
    product; an all-zero dense part is scipy's CSR product."""
    import scipy.sparse as sp
    rng = np.random.default_rng(3)
    p = random_problem(rng, 7, 48, 3, "affine", 2)
    y, bd = orc.gemv(p, x=np.zeros((2, 48), np.uint16))
    assert np.all(y == 0) and np.all(bd == 0)
    wd = np_h2d(orc.decode(p))
    hit = np.zeros(48, bool)
    hit[p.col_idx] = True
    j = int(np.flatnonzero(~hit)[0])
    e = np.zeros((1, 48), np.uint16)
    e[0, j] = 0x3C00
    y, _ = orc.gemv(p, x=e)
    assert np.array_equal(y[0], wd[:, j])
    empty = types.SimpleNamespace(**vars(p))
    empty.row_ptr = np.zeros(8, np.int32)
    empty.col_idx = np.zeros(0, np.int32)
    empty.values = np.zeros(0, np.uint16)
    y_dense, _ = orc.gemv(empty)
    xd = np_h2d(p.x)
    assert np.allclose(y_dense, xd @ wd.T, rtol=0, atol=1e-12 * (np.abs(xd) @ np.abs(wd).T).max())
    zero_dense = types.SimpleNamespace(**vars(p))
    zero_dense.codes = np.repeat(np_h2d(p.zeros).astype(np.uint8), 16, axis=1)
    y_sp, _ = orc.gemv(zero_dense)
    A = sp.csr_matrix((np_h2d(p.values), p.col_idx, p.row_ptr), shape=(7, 48))
    want = np.stack([A @ xd[b] for b in range(2)])
    assert np.allclose(y_sp, want, rtol=1e-15, atol=0)


def pin_decomposition(orc):
    """What - W_dense is the CSR matrix: zero off the outliers, the fp16 value
    on them (a sum of two fp16 values is exact in fp64)."""
    rng = np.random.default_rng(9)
    for mode in ("lut", "affine"):
        p = random_problem(rng, 9, 64, 4, mode, 1, nnz_per_row_max=9)
        diff = orc.materialize(p) - np_h2d(orc.decode(p))
        want = np.zeros_like(diff)
        for i in range(p.rows):
            for k in range(p.row_ptr[i], p.row_ptr[i + 1]):
                want[i, p.col_idx[k]] = np_h2d(p.values[k])
        assert np.array_equal(diff, want)


def pin_rows_subset(orc):
    """Sampled rows equal the same rows of the full product."""
    p = synth.make_problem(33, 64, 3, "affine", 0.05, "uniform", 1, 2)
    y, bd = orc.gemv(p)
    rows = [32, 0, 17, 17]
    ys, bs = orc.gemv(p, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(bs, bd[:, rows])


PINS = [pin_half_to_double_exhaustive, pin_double_to_half, pin_csr_example,
        pin_lut_decode_identity, pin_affine_decode_golden, pin_affine_group_layout,
        pin_bitplane_decode_golden, pin_bitplane_group_layout, pin_bitplane_uniform_grid_is_affine,
        pin_two_axis_golden, pin_two_axis_unit_scales, pin_intgrid_decode_golden, pin_intgrid_group_layout,
        pin_gemv_exact, pin_special_cases, pin_decomposition, pin_rows_subset]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


# Each entry plants one plausible mistake in a copy of oracle.c.
MUTANTS = {
    "drop_sparse_term": ("wrow[col_idx[k]] += oracle_half_to_double(values[k]);",
                         "wrow[col_idx[k]] += 0.0;"),
    "sparse_sign": ("wrow[col_idx[k]] += oracle_half_to_double(values[k]);",
                    "wrow[col_idx[k]] -= oracle_half_to_double(values[k]);"),
    "sparse_column": ("wrow[col_idx[k]] += oracle_half_to_double(values[k]);",
                      "wrow[k - row_ptr[i]] += oracle_half_to_double(values[k]);"),
    "skip_first_outlier": ("for (int64_t k = row_ptr[i]; k < row_ptr[i + 1]; k++)",
                           "for (int64_t k = row_ptr[i] + 1; k < row_ptr[i + 1]; k++)"),
    "affine_zero_sign": ("scale * ((double)q - zero)", "scale * ((double)q + zero)"),
    "affine_group_width": ("j / ORACLE_GROUP;", "j / 8;"),
    "lut_row_index": ("return table[i * ((int64_t)1 << bits) + q];", "return table[q];"),
    "ties_not_even": ("if (r > 0.5 || (r == 0.5 && (n & 1)))", "if (r > 0.5)"),
    "ties_away": ("if (r > 0.5 || (r == 0.5 && (n & 1)))", "if (r >= 0.5)"),
    "subnormal_binade": ("if (E < -14)\n        E = -14;", "if (E < -15)\n        E = -15;"),
    "overflow_edge": ("if (E > 15)\n        return sign | 0x7C00;",
                      "if (E > 16)\n        return sign | 0x7C00;"),
    "half_bias": ("ldexp((double)(1024 + m), e - 25)", "ldexp((double)(1024 + m), e - 24)"),
    "half_subnormal": ("ldexp((double)m, -24)", "ldexp((double)m, -25)"),
    "bound_signed": ("mag += fabs(wrow[j]) * fabs(xd[(int64_t)b * cols + j]);",
                     "mag += wrow[j] * xd[(int64_t)b * cols + j];"),
    "x_transposed": ("acc += wrow[j] * xd[(int64_t)b * cols + j];",
                     "acc += wrow[j] * xd[(int64_t)j * batch + b];"),
    "dropped_x": ("acc += wrow[j] * xd[(int64_t)b * cols + j];", "acc += wrow[j];"),
    "bitplane_bit_order": ("if ((q >> (p - 1)) & 1)", "if ((q >> p) & 1)"),
    "bitplane_drop_bias": ("double w = oracle_half_to_double(c[0]);", "double w = 0.0;"),
    "bitplane_group_size": ("int64_t gsize = (int64_t)32 << bits;", "int64_t gsize = (int64_t)16 << bits;"),
    "bitplane_round_each_step": ("                w += oracle_half_to_double(c[p]);",
                                 "                w = oracle_half_to_double(oracle_double_to_half(w + oracle_half_to_double(c[p])));"),
    "bitplane_coef_row_stride": ("table + (i * (cols / gsize) + j / gsize) * (bits + 1)",
                                 "table + (j / gsize) * (bits + 1)"),
    "two_axis_scaled_outliers": ("        wrow[col_idx[k]] += oracle_half_to_double(values[k]);\n}\n\nvoid oracle_weight_row(",
                                 "        wrow[col_idx[k]] += r * oracle_half_to_double(values[k]);\n}\n\nvoid oracle_weight_row("),
    "two_axis_col_by_row": ("double c = cscale ? oracle_half_to_double(cscale[j]) : 1.0;",
                            "double c = cscale ? oracle_half_to_double(cscale[i]) : 1.0;"),
    "two_axis_no_row_scale": ("double r = rscale ? oracle_half_to_double(rscale[i]) : 1.0;", "double r = 1.0;"),
    "intgrid_unsigned": ("int qi = ((const int16_t *)codes)[i * (int64_t)cols + j];",
                         "int qi = ((const uint16_t *)codes)[i * (int64_t)cols + j];"),
    "intgrid_group_width": ("table[i * (int64_t)(cols / ORACLE_GROUP) + j / ORACLE_GROUP]);\n        return oracle_double_to_half(scale * (double)qi);",
                            "table[i * (int64_t)(cols / ORACLE_GROUP) + j / 32]);\n        return oracle_double_to_half(scale * (double)qi);"),
    "first_column_skipped": ("for (int64_t j = 0; j < cols; j++) {\n                acc",
                             "for (int64_t j = 1; j < cols; j++) {\n                acc"),
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
