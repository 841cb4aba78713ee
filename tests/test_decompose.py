"""dsq_decompose: the on-device outlier selection, CSR build and quantization
must give, bit for bit, the oracle's decomposition of the same fp32 weights
(every output array), and the matrix it produces must multiply like the
oracle's.  Host-side argument checks run without a GPU."""
import ctypes

import numpy as np
import pytest

import dense_sparse_quantized_b200 as dsq
import synth

torch = pytest.importorskip("torch")

TOL = 1e-3


def test_decompose_workspace_query_and_refusals():
    lib = dsq.library()
    size = ctypes.c_size_t(0)
    d = dsq.Desc(11008, 4096, 3, dsq.MODE_AFFINE_G16, 450888)
    assert lib.dsq_decompose(ctypes.byref(d), None, None, None, None, None, None, None, None,
                             ctypes.byref(size), None) == dsq.DSQ_ERR_BUFFER_TOO_SMALL
    assert size.value >= 11008 * 4096 // 8
    assert lib.dsq_decompose(None, None, None, None, None, None, None, None, None,
                             ctypes.byref(size), None) == dsq.DSQ_ERR_INVALID_ARG
    for desc, rc in ((dsq.Desc(64, 512, 3, dsq.MODE_BITPLANE, 0), dsq.DSQ_ERR_UNSUPPORTED),
                     (dsq.Desc(64, 40000, 3, dsq.MODE_LUT_ROW, 0), dsq.DSQ_ERR_UNSUPPORTED),
                     (dsq.Desc(64, 40, 3, dsq.MODE_AFFINE_G16, 0), dsq.DSQ_ERR_INVALID_ARG),
                     (dsq.Desc(64, 64, 3, dsq.MODE_AFFINE_G16, 64 * 64 + 1), dsq.DSQ_ERR_INVALID_ARG)):
        assert lib.dsq_decompose(ctypes.byref(desc), None, None, None, None, None, None, None, None,
                                 ctypes.byref(size), None) == rc


def _cases():
    rng = np.random.default_rng(12)
    ties = (rng.integers(-3, 4, (40, 96)) / 8.0).astype(np.float32)   # massive ties at every |w|
    zero_rows = synth.spiky_weights(30, 64, 0.05, 13)
    zero_rows[[3, 17]] = 0.0                                          # degenerate groups
    one_row = synth.spiky_weights(1, 16, 0.0, 14)
    heavy = synth.spiky_weights(20, 128, 0.01, 15)
    heavy[7] = 5.0 + np.arange(128, dtype=np.float32)                 # a row made only of outliers
    return [
        ("c0 shape, table 3-bit, 1% outliers", synth.spiky_weights(1024, 1024, 0.01, 0), 3, "lut", 10486),
        ("c2 shape, affine 3-bit, 1% outliers", synth.spiky_weights(11008, 4096, 0.01, 2), 3, "affine", 450888),
        ("c3 shape, table 4-bit, 0.5% outliers", synth.spiky_weights(4096, 11008, 0.005, 3), 4, "lut", 225444),
        ("ties, affine", ties, 3, "affine", 700), ("ties, table", ties, 4, "lut", 1000),
        ("zero rows, affine", zero_rows, 4, "affine", 40), ("zero rows, table", zero_rows, 3, "lut", 40),
        ("no outliers", heavy, 3, "affine", 0), ("all outliers", heavy[:2, :32].copy(), 3, "affine", 64),
        ("one group", one_row, 3, "affine", 1), ("a row of outliers, table", heavy, 3, "lut", 140),
    ]


CASES = _cases()


@pytest.mark.gpu
@pytest.mark.parametrize("case", range(len(CASES)), ids=[c[0] for c in CASES])
def test_decompose_bit_exact(orc, case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    what, w, bits, mode, nnz = CASES[case]
    out = dsq.decompose(torch.from_numpy(w).cuda(), bits, mode, nnz)
    torch.cuda.synchronize()
    got = [None if t is None else t.cpu().numpy() for t in out]
    want = orc.decompose(w, bits, mode, nnz)
    names = ("codes", "table", "zeros", "row_ptr", "col_idx", "values")
    for name, g, e in zip(names, got, want):
        if e is None:
            assert g is None, (what, name)
            continue
        g = g.view(np.uint16) if g.dtype == np.float16 else g
        assert g.shape == e.shape and np.array_equal(g, e), (what, name, int(np.count_nonzero(g != e)))


@pytest.mark.gpu
@pytest.mark.parametrize("mode,bits", [("affine", 3), ("lut", 4)])
def test_decompose_then_product(orc, mode, bits):
    """Weights decomposed on the device, packed and multiplied: y against the
    oracle's product of the same arrays."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import types
    w = synth.spiky_weights(2048, 1024, 0.01, 21)
    nnz = round(0.01 * w.size)
    codes, table, zeros, rp, ci, va = [None if t is None else t.cpu().numpy() for t in
                                       dsq.decompose(torch.from_numpy(w).cuda(), bits, mode, nnz)]
    h16 = lambda a: None if a is None else a.view(np.uint16)  # noqa: E731
    rng = np.random.default_rng(22)
    p = types.SimpleNamespace(rows=w.shape[0], cols=w.shape[1], bits=bits, mode=mode, codes=codes,
                              table=h16(table), zeros=h16(zeros), row_ptr=rp, col_idx=ci, values=h16(va),
                              x=synth.f16_bits(rng.standard_normal((2, w.shape[1]))))
    with dsq.Handle(dsq.pack_problem(p)) as h:
        x = torch.from_numpy(p.x.view(np.int16)).view(torch.float16).cuda()
        y = h.gemv(x)
        torch.cuda.synchronize()
        yv = y.cpu().view(torch.int16).numpy().view(np.float16).astype(np.float64)
    y_ref, bound = orc.gemv(p)
    assert np.all(np.abs(yv - y_ref) <= TOL * bound)
