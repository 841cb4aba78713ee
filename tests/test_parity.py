"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Decode: the device's decoded W_dense is bit-identical to the oracle's.
Product: |y - y_ref| <= 1e-3 * bound element by element, bound =
sum_j |What[i][j]| * |x[b][j]|; where bound is 0, y is exactly 0.  The
tolerance covers the fp16 rounding of y (<= 2^-11 |y|), the use of exact
rather than fp16-rounded affine weights inside the group sums (<= 2^-11 per
weight, i.e. <= 4.9e-4 * bound) and fp32 accumulation.
"""
import os

import numpy as np
import pytest

import dense_sparse_quantized_b200 as dsq
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def to_dev(bits: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()


def to_bits(t) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check_y(y_bits, y_ref, bound, what=""):
    y = y_bits.view(np.float16).astype(np.float64)
    assert np.all(np.isfinite(y)), what
    zero = bound == 0
    assert np.all(y[zero] == 0), what
    if (~zero).any():
        ratio = np.abs(y[~zero] - y_ref[~zero]) / bound[~zero]
        assert ratio.max() <= TOL, (what, float(ratio.max()))
        return float(ratio.max())
    return 0.0


def gemv(h, x_bits, batch):
    x = to_dev(x_bits[:batch])
    y = h.gemv(x)
    torch.cuda.synchronize()
    h.check()
    return to_bits(y)


_cache = {}


def config(name):
    if name not in _cache:
        p = synth.make_config(name)
        _cache[name] = (p, dsq.Handle(dsq.pack_problem(p)))
    return _cache[name]


def sample_rows(p, n=768, seed=0):
    """A sample of rows that always holds the first, the last and the rows
    with the most outliers, plus random ones."""
    rng = np.random.default_rng(seed)
    counts = np.diff(p.row_ptr)
    heavy = np.argsort(-counts, kind="stable")[:64]
    rnd = rng.choice(p.rows, min(n, p.rows), replace=False)
    return np.unique(np.concatenate([[0, p.rows - 1], heavy, rnd])).astype(np.int32)


# ------------------------------------------------------------- full-size configs

SMALL_CONFIGS = ["c0", "c1", "c2", "c3"]
C4 = ["c4_" + n for n, _, _ in synth.C4_LAYERS]
BITPLANE = ["bp2", "bp3"]


@pytest.mark.parametrize("name", SMALL_CONFIGS + C4 + BITPLANE)
def test_decode_bit_exact(orc, name):
    p, h = config(name)
    got = to_bits(h.decode())
    want = orc.decode(p)
    mism = np.count_nonzero(got != want)
    assert mism == 0, f"{mism} decoded weights differ"


@pytest.mark.parametrize("name,batch", [("c0", 1), ("c1", 1), ("c2", 1), ("c3", 1), ("c3", 2),
                                        ("c3", 4), ("c3", 8)])
def test_gemv_full_oracle(orc, name, batch):
    p, h = config(name)
    y = gemv(h, p.x, batch)
    y_ref, bound = orc.gemv(p, x=p.x[:batch])
    check_y(y, y_ref, bound, f"{name} B={batch}")


def oracle_all_rows(orc, p, x):
    """The oracle over every row, computed on row slices in parallel threads
    (its C entry point releases the GIL); same values as one call."""
    from concurrent.futures import ThreadPoolExecutor
    slices = np.array_split(np.arange(p.rows, dtype=np.int32), max(1, min(16, os.cpu_count() or 1)))
    with ThreadPoolExecutor(max_workers=len(slices)) as pool:
        parts = list(pool.map(lambda r: orc.gemv(p, x=x, rows=r), slices))
    return np.concatenate([a for a, _ in parts], axis=1), np.concatenate([b for _, b in parts], axis=1)


@pytest.mark.parametrize("name", BITPLANE)
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5])
def test_gemv_bitplane_every_row(orc, name, batch):
    """BPDQ matrices (11008 x 4096, 2 and 3 planes, 1% outliers): the batch-1
    table kernel with per-group levels, the 2-4 row kernel, and both for 5
    rows; every row against the oracle."""
    p, h = config(name)
    xb = synth.f16_bits(np.random.default_rng(batch).standard_normal((batch, p.cols)))
    y = gemv(h, xb, batch)
    y_ref, bound = oracle_all_rows(orc, p, xb)
    check_y(y, y_ref, bound, f"{name} B={batch}")


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("rows,cols", [(1, 256), (7, 1024), (33, 4096), (130, 512), (64, 24576), (5, 25600)])
def test_bitplane_small_shapes(orc, bits, rows, cols):
    """Ragged row counts, one group per row up to 96 groups; 25600 columns
    exceed the tuned kernels' 24 column warps and run the generic kernel."""
    G = synth.bitplane_group(bits)
    cols = max(G, cols // G * G)
    p = synth.make_problem(rows, cols, bits, "bitplane", 0.02, "uniform", rows + bits, 3)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        assert np.array_equal(to_bits(h.decode()), orc.decode(p))
        for batch in (1, 2, 3):
            y = gemv(h, p.x, batch)
            y_ref, bound = orc.gemv(p, x=p.x[:batch])
            check_y(y, y_ref, bound, f"{rows}x{cols} bitplane k={bits} B={batch}")


@pytest.mark.parametrize("batch", [1, 2, 5, 9])
def test_gemv_intgrid_every_row(orc, batch):
    """Huffman-coded integer grid (11008 x 4096, spikes in the grid): the
    variable-length-decode kernel, every row against the oracle; the decode
    is bit-exact."""
    p, h = config("hq")
    if batch == 1:
        assert np.array_equal(to_bits(h.decode()), orc.decode(p))
    xb = synth.f16_bits(np.random.default_rng(80 + batch).standard_normal((batch, p.cols)))
    y = gemv(h, xb, batch)
    y_ref, bound = oracle_all_rows(orc, p, xb)
    check_y(y, y_ref, bound, f"hq B={batch}")


def test_intgrid_small_cases(orc):
    """Long codes (past the fast table), one-symbol codes, extra CSR
    outliers, ragged row counts, the widest row (65520 columns: x of one
    activation row fills the kernel's shared-memory stage)."""
    import types
    rng = np.random.default_rng(9)
    for rows, cols in ((1, 16), (7, 48), (33, 4096), (130, 512), (2, 65520)):
        q = (np.minimum(rng.geometric(0.4, (rows, cols)) - 1, 60) * np.where(rng.random((rows, cols)) < 0.5, -1, 1)).astype(np.int16)
        q.reshape(-1)[0] = 8191
        sc = synth.f16_bits(np.exp2(rng.integers(-12, 0, (rows, cols // 16))))
        base = synth.make_problem(rows, cols, 3, "affine", 0.02, "uniform", rows, 3)
        p = types.SimpleNamespace(rows=rows, cols=cols, bits=14, mode="intgrid", codes=q, table=sc, zeros=None,
                                  row_ptr=base.row_ptr, col_idx=base.col_idx, values=base.values, x=base.x)
        with dsq.Handle(dsq.pack_problem(p)) as h:
            assert np.array_equal(to_bits(h.decode()), orc.decode(p))
            for batch in (1, 3):
                y = gemv(h, p.x, batch)
                y_ref, bound = orc.gemv(p, x=p.x[:batch])
                check_y(y, y_ref, bound, f"intgrid {rows}x{cols} B={batch}")
    p = types.SimpleNamespace(rows=3, cols=64, bits=14, mode="intgrid", codes=np.full((3, 64), 5, np.int16),
                              table=np.full((3, 4), 0x3800, np.uint16), zeros=None, row_ptr=np.zeros(4, np.int32),
                              col_idx=np.zeros(0, np.int32), values=np.zeros(0, np.uint16),
                              x=synth.f16_bits(rng.standard_normal((1, 64))))
    with dsq.Handle(dsq.pack_problem(p)) as h:
        assert np.array_equal(to_bits(h.decode()), orc.decode(p))
        y_ref, bound = orc.gemv(p)
        check_y(gemv(h, p.x, 1), y_ref, bound, "one symbol")


@pytest.mark.parametrize("batch", [1, 2])
def test_gemv_two_axis_every_row(orc, batch):
    """SINQ two-axis scales around a 3-bit table matrix (11008 x 4096): the
    batch-1 table kernel with x times c formed in fp32 and r applied per
    row; every row against the oracle; the decode is the unscaled W_dense."""
    p, h = config("sq3")
    if batch == 1:
        assert np.array_equal(to_bits(h.decode()), orc.decode(p))
    xb = synth.f16_bits(np.random.default_rng(70 + batch).standard_normal((batch, p.cols)))
    y = gemv(h, xb, batch)
    y_ref, bound = oracle_all_rows(orc, p, xb)
    check_y(y, y_ref, bound, f"sq3 B={batch}")


@pytest.mark.parametrize("bits,mode,cols", [(3, "lut", 1024), (4, "lut", 512), (3, "affine", 1024),
                                            (4, "affine", 512), (2, "bitplane", 512), (3, "bitplane", 1024),
                                            (3, "lut", 25600)])
def test_two_axis_all_modes(orc, bits, mode, cols):
    """Two-axis scales on every mode and through every path that serves them
    (batch-1 table kernel, the generic kernel for affine matrices, past 24
    column warps and for more rows), batches 1-3 and 9."""
    p = synth.make_problem(37, cols, bits, mode, 0.02, "uniform", bits + cols, 9, two_axis=True)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        assert np.array_equal(to_bits(h.decode()), orc.decode(p))
        for batch in (1, 2, 3, 9):
            y = gemv(h, p.x, batch)
            y_ref, bound = orc.gemv(p, x=p.x[:batch])
            check_y(y, y_ref, bound, f"two-axis {bits} {mode} {cols} B={batch}")


@pytest.mark.parametrize("name", C4)
@pytest.mark.parametrize("batch", [1, 16])
def test_gemv_c4_every_row(orc, name, batch):
    p, h = config(name)
    y = gemv(h, p.x, batch)
    y_ref, bound = oracle_all_rows(orc, p, p.x[:batch])
    check_y(y, y_ref, bound, f"{name} B={batch}")


# ------------------------------------------------------------- small shapes

SHAPES = [(1, 16), (7, 48), (64, 1024), (7, 16), (1, 1024), (64, 48), (33, 4096), (130, 80)]


@pytest.mark.parametrize("bits,mode", [(3, "lut"), (4, "lut"), (3, "affine"), (4, "affine")])
@pytest.mark.parametrize("rows,cols", SHAPES)
def test_small_shapes(orc, bits, mode, rows, cols):
    p = synth.make_problem(rows, cols, bits, mode, 0.02, "uniform", rows * 7 + cols, 3)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        assert np.array_equal(to_bits(h.decode()), orc.decode(p))
        for batch in (1, 2, 3):
            y = gemv(h, p.x, batch)
            y_ref, bound = orc.gemv(p, x=p.x[:batch])
            check_y(y, y_ref, bound, f"{rows}x{cols} {bits} {mode} B={batch}")


@pytest.mark.parametrize("mode", ["lut", "affine"])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8, 15, 16, 17, 31, 32, 40])
def test_batches(orc, mode, batch):
    p = synth.make_problem(96, 272, 3, mode, 0.02, "uniform", 123, batch)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        y = gemv(h, p.x, batch)
        y_ref, bound = orc.gemv(p)
        check_y(y, y_ref, bound, f"{mode} B={batch}")


@pytest.mark.parametrize("rows,cols", [(37, 272), (130, 1024), (16, 11008)])
@pytest.mark.parametrize("batch", [2, 3, 7, 8, 9, 16, 17, 33])
def test_table4_tensor_core_batches(orc, rows, cols, batch):
    """4-bit row tables from 2 activation rows on: the centroids looked up
    into warp-level MMA fragments (8 activation rows per launch up to 8,
    then 16 per launch).  Ragged 16-row tiles, an odd slot count with a
    16-column tail slot (272 columns), c3's width."""
    p = synth.make_problem(rows, cols, 4, "lut", 0.02, "uniform", rows + cols + batch, batch)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        y = gemv(h, p.x, batch)
        y_ref, bound = orc.gemv(p)
        check_y(y, y_ref, bound, f"table4 {rows}x{cols} B={batch}")


@pytest.mark.parametrize("batch", [4, 16])
def test_table4_tile_with_many_outlier_rounds(orc, batch):
    """The first 16-row tile has an outlier on every column of every row
    (16 x 16384 entries: 2048 warp pieces of 128 entries), more than one
    round of piece sums holds, so the sums are folded over several rounds;
    the rows after it keep a few outliers."""
    p = synth.make_problem(40, 16384, 4, "lut", 0.001, "uniform", 12, batch)
    rng = np.random.default_rng(3)
    rows = [np.arange(p.cols) if i < 16 else p.col_idx[p.row_ptr[i]:p.row_ptr[i + 1]] for i in range(p.rows)]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    q = edited(p, row_ptr=rp, col_idx=ci, values=synth.f16_bits(rng.laplace(0, 0.2, ci.size)))
    with dsq.Handle(dsq.pack_problem(q)) as h:
        y = gemv(h, q.x, batch)
    y_ref, bound = orc.gemv(q)
    check_y(y, y_ref, bound, f"table4 many outlier rounds B={batch}")


# ------------------------------------------------------------- edge cases

def edited(p, **kw):
    import dataclasses
    return dataclasses.replace(p, **kw)


@pytest.mark.parametrize("mode", ["lut", "affine"])
def test_empty_csr(orc, mode):
    p = synth.make_problem(50, 256, 3, mode, 0.0, "none", 4, 2)
    assert p.nnz == 0
    with dsq.Handle(dsq.pack_problem(p)) as h:
        y_ref, bound = orc.gemv(p)
        check_y(gemv(h, p.x, 2), y_ref, bound, "empty csr")


@pytest.mark.parametrize("mode", ["lut", "affine"])
def test_all_outlier_rows(orc, mode):
    """Row 3 has an outlier on every column (nnz = N); row 10 likewise; the
    other rows keep their outliers."""
    p = synth.make_problem(20, 96, 4, mode, 0.01, "uniform", 5, 2)
    rng = np.random.default_rng(1)
    rows = []
    for i in range(p.rows):
        if i in (3, 10):
            rows.append(np.arange(96))
        else:
            rows.append(p.col_idx[p.row_ptr[i]:p.row_ptr[i + 1]])
    counts = np.array([len(r) for r in rows])
    rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    va = synth.f16_bits(rng.laplace(0, 0.2, ci.size))
    q = edited(p, row_ptr=rp, col_idx=ci, values=va)
    with dsq.Handle(dsq.pack_problem(q)) as h:
        y_ref, bound = orc.gemv(q)
        check_y(gemv(h, q.x, 2), y_ref, bound, "all-outlier rows")


@pytest.mark.parametrize("batch", [16, 32, 40])
def test_tile_outliers_staged_and_not(orc, batch):
    """Tensor-core path: the first 128-row tile holds 300 outliers per row, more
    than the CSR slice kept in shared memory, so its outlier warps read the
    entries from global memory; the other tiles (the last one ragged) are
    staged.  Both must match the oracle."""
    p = synth.make_problem(300, 2048, 3, "affine", 0.01, "uniform", 77, batch)
    rng = np.random.default_rng(2)
    rows = []
    for i in range(p.rows):
        if i < 128:
            rows.append(np.sort(rng.choice(p.cols, 300, replace=False)))
        else:
            rows.append(p.col_idx[p.row_ptr[i]:p.row_ptr[i + 1]])
    counts = np.array([len(r) for r in rows])
    rp = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    va = synth.f16_bits(rng.laplace(0, 0.2, ci.size))
    q = edited(p, row_ptr=rp, col_idx=ci, values=va)
    with dsq.Handle(dsq.pack_problem(q)) as h:
        y_ref, bound = orc.gemv(q)
        check_y(gemv(h, q.x, batch), y_ref, bound, f"staged and unstaged tiles B={batch}")


@pytest.mark.parametrize("name", ["c2", "c3"])
def test_zero_and_one_hot_x(orc, name):
    p, h = config(name)
    x0 = np.zeros((1, p.cols), np.uint16)
    y = gemv(h, x0, 1).view(np.float16)
    assert np.all(y == 0)
    hit = np.zeros(p.cols, bool)
    hit[p.col_idx] = True
    j = int(np.flatnonzero(~hit)[0]) if (~hit).any() else 0
    e = np.zeros((1, p.cols), np.uint16)
    e[0, j] = 0x3C00
    y = gemv(h, e, 1)
    y_ref, bound = orc.gemv(p, x=e)
    check_y(y, y_ref, bound, "one-hot")
    if not hit[j]:
        # y_i = W_dense[i][j] exactly: one product, no rounding beyond fp16.
        wd = orc.decode(p)[:, j]
        assert np.array_equal(y[0].view(np.float16).astype(np.float64),
                              wd.view(np.float16).astype(np.float64))


def test_degenerate_shapes():
    for rows, cols in ((0, 32), (5, 0)):
        blob = dsq.pack(rows, cols, 3, "affine", np.zeros((rows, cols), np.uint8),
                        np.zeros((rows, cols // 16), np.uint16),
                        np.zeros((rows, cols // 16), np.uint16), np.zeros(rows + 1, np.int32),
                        np.zeros(0, np.int32), np.zeros(0, np.uint16))
        with dsq.Handle(blob) as h:
            x = torch.randn(2, max(cols, 1), device="cuda").half()[:, :cols].contiguous()
            y = torch.full((2, rows), 7.0, device="cuda").half()
            h.gemv(x if cols else torch.empty((2, 0), device="cuda", dtype=torch.float16), y)
            torch.cuda.synchronize()
            assert torch.all(y == 0)


def test_y_written_in_place_only(orc):
    """y is written exactly in its [batch, rows] box: guard bytes around it
    stay untouched."""
    p = synth.make_problem(37, 160, 3, "affine", 0.03, "uniform", 8, 3)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        buf = torch.full((3 * 37 + 64,), 123.0, device="cuda").half()
        y = buf[32:32 + 3 * 37].view(3, 37)
        x = to_dev(p.x)
        h.gemv(x, y)
        torch.cuda.synchronize()
        b = buf.cpu()
        assert torch.all(b[:32] == 123.0) and torch.all(b[32 + 3 * 37:] == 123.0)
        y_ref, bound = orc.gemv(p)
        check_y(to_bits(y), y_ref, bound)


def test_misaligned_pointers_rejected():
    p = synth.make_problem(8, 64, 3, "affine", 0.02, "uniform", 1, 1)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        buf = torch.zeros(200, device="cuda", dtype=torch.float16)
        rc = dsq.library().dsq_gemv(h._h, buf.data_ptr() + 2, buf.data_ptr() + 256, 1, None)
        assert rc == dsq.DSQ_ERR_INVALID_ARG


def test_streams_and_repeat_calls_agree():
    p, h = config("c2")
    x = to_dev(p.x[:1])
    s = torch.cuda.Stream()
    y0 = h.gemv(x)
    with torch.cuda.stream(s):
        y1 = h.gemv(x, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


@pytest.mark.parametrize("mode,bits,batch", [("affine", 3, 1), ("affine", 3, 16), ("lut", 3, 1), ("lut", 3, 4),
                                            ("lut", 4, 4), ("lut", 4, 16)])
def test_back_to_back_calls_read_the_x_just_written(mode, bits, batch):
    """The kernels start before the previous kernel in the stream ends
    (programmatic dependent launch) and must still read the x that kernel
    wrote and write y after it: x is rewritten by a copy kernel right before
    every call, with no synchronisation, and each y must equal, bit for bit,
    the y of the same x computed in isolation."""
    p = synth.make_problem(1024, 2048, bits, mode, 0.01, "uniform", 31, batch)
    rng = np.random.default_rng(5)
    xs = [to_dev(synth.f16_bits(rng.standard_normal((batch, p.cols)))) for _ in range(6)]
    with dsq.Handle(dsq.pack_problem(p)) as h:
        ref = []
        for xv in xs:
            ref.append(h.gemv(xv).clone())
            torch.cuda.synchronize()
        x = torch.empty_like(xs[0])
        y = torch.empty((batch, p.rows), dtype=torch.float16, device="cuda")
        got = []
        for _ in range(3):
            for xv in xs:
                x.copy_(xv)        # a kernel writes x ...
                h.gemv(x, y)       # ... and the product reads it at once
                got.append(y.clone())
        torch.cuda.synchronize()
        h.check()
    for i, g in enumerate(got):
        assert torch.equal(g.view(torch.int16), ref[i % len(xs)].view(torch.int16)), i


# ------------------------------------------------------------- wide-range activations

F16_OVERFLOW = 65520.0   # |v| at or above this rounds to inf in fp16


def zero_columns(p, cols):
    """p with What[:, cols] == 0 exactly: every code there set to its group's
    zero point (the dense weight decodes to 0, as at a hole) and the outliers
    on those columns dropped."""
    codes = p.codes.copy()
    z = p.zeros.view(np.float16).astype(np.uint8)
    codes[:, cols] = z[:, cols // synth.GROUP]
    keep = ~np.isin(p.col_idx, cols)
    rows = np.repeat(np.arange(p.rows), np.diff(p.row_ptr))[keep]
    rp = np.concatenate([[0], np.cumsum(np.bincount(rows, minlength=p.rows))]).astype(np.int32)
    return edited(p, codes=codes, row_ptr=rp, col_idx=p.col_idx[keep].astype(np.int32),
                  values=p.values[keep])


def wide_problem(p, batch, per_group, seed, big=60000.0, small=1e-4):
    """The matrix with exact zeros on a few columns, and activations spanning
    the fp16 range: +-`big` on those columns, |x| ~ `small` everywhere else.
    The large entries add nothing to y or to the error bound, so a kernel
    whose rounding error follows them (a zero point subtracted after the
    group sum, say) shows it.  per_group False: 3 columns; True: one column
    in every group of 16."""
    rng = np.random.default_rng(seed)
    if per_group:
        cols = np.arange(0, p.cols, synth.GROUP) + rng.integers(0, synth.GROUP, p.cols // synth.GROUP)
    else:
        cols = np.sort(rng.choice(p.cols, 3, replace=False))
    q = zero_columns(p, cols)
    x = small * (1.0 + rng.random((batch, p.cols))) * rng.choice([-1.0, 1.0], (batch, p.cols))
    x[:, cols] = big * rng.choice([-1.0, 1.0], (batch, cols.size))
    return q, synth.f16_bits(x)


@pytest.mark.parametrize("per_group", [False, True])
@pytest.mark.parametrize("batch", [1, 2, 3, 16])
def test_wide_range_x_c2(orc, per_group, batch):
    """c2 (11008 x 4096, 3-bit affine) with activations near +-6e4 on columns
    where every weight is exactly 0 and ~1e-4 elsewhere, through every path
    an affine 3-bit matrix takes (batch-1 kernel, once per row at batch 2,
    tensor cores from batch 3 / 16); every row against the oracle."""
    p, _ = config("c2")
    q, xb = wide_problem(p, batch, per_group, 40 + batch)
    with dsq.Handle(dsq.pack_problem(q)) as h:
        y = gemv(h, xb, batch)
    y_ref, bound = orc.gemv(q, x=xb)
    check_y(y, y_ref, bound, f"c2 wide-range x per_group={per_group} B={batch}")


@pytest.mark.parametrize("rows,cols", [(256, 1024), (130, 4096), (64, 24640)])
@pytest.mark.parametrize("per_group", [False, True])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_wide_range_x_small_affine(orc, rows, cols, per_group, batch):
    """Small affine 3-bit shapes with the same activations; 24640 columns
    exceed the batch-1 kernel's 24 column groups and run the generic
    kernel."""
    p = synth.make_problem(rows, cols, 3, "affine", 0.01, "uniform", rows + cols, 1)
    q, xb = wide_problem(p, batch, per_group, 7 * batch + rows)
    with dsq.Handle(dsq.pack_problem(q)) as h:
        y = gemv(h, xb, batch)
    y_ref, bound = orc.gemv(q, x=xb)
    check_y(y, y_ref, bound, f"{rows}x{cols} wide-range per_group={per_group} B={batch}")


# ------------------------------------------------------------- bounded waits

def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable(orc):
    """A kernel waits on a barrier nothing arrives on, through the bounded wait
    every pipeline uses: after about 2 s it gives up and sets the status word;
    dsq_check reports DSQ_ERR_DEVICE once and clears it; the next product on
    the same handle is correct and checks clean."""
    import time
    p = synth.make_problem(64, 512, 3, "affine", 0.01, "uniform", 11, 1)
    with dsq.Handle(dsq.pack_problem(p)) as h:
        t0 = time.perf_counter()
        h.selftest_wait_timeout()
        with pytest.raises(dsq.DSQError) as e:
            h.check()
        assert e.value.status == dsq.DSQ_ERR_DEVICE
        assert time.perf_counter() - t0 >= 1.0   # the wait ran to its limit
        h.check()                                 # the word was cleared
        y = gemv(h, p.x, 1)
        y_ref, bound = orc.gemv(p)
        check_y(y, y_ref, bound, "after a timed-out wait")
