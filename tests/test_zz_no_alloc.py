"""dsq_gemv_noalloc: the handle-free product for callers that may not
allocate device memory (a plugin whose buffers all come from its host
program's pool, or code where cudaMalloc's implicit synchronisation is not
allowed).

The caller uploads the packed blob into memory it owns; the library's
kernels keep their scratch in one fixed array.  This file runs last so that a
failure here comes after every other test has run.  Each check compares the
entry point's y with dsq_gemv's (a handle on the same blob) element by
element, within the parity tolerance 1e-3 * sum_j |What[i][j]| |x[b][j]| of
the other GPU tests, on two calls in a row that leave different contents in
the shared scratch (two matrices with different K splits, two inputs).
"""
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


def to_f64(t) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16).view(np.float16).astype(np.float64)


def upload(blob: bytes):
    """The caller's own device copy of the blob (the test allocates it; the
    entry point never does)."""
    return torch.frombuffer(bytearray(blob), dtype=torch.uint8).cuda()


def within(y_new, y_old, bound, what):
    assert np.all(np.isfinite(y_new)), what
    zero = bound == 0
    assert np.all(y_new[zero] == y_old[zero]), what
    ratio = np.abs(y_new[~zero] - y_old[~zero]) / bound[~zero]
    assert ratio.max(initial=0.0) <= TOL, (what, float(ratio.max(initial=0.0)))


def random_x(seed, batch, cols):
    rng = np.random.default_rng(seed)
    return synth.f16_bits(rng.standard_normal((batch, cols)))


# Affine 3-bit matrices with different row counts, so consecutive calls leave
# different contents in the shared scratch: 2000 rows (16 tiles of 128 rows)
# and 6000 rows (47 tiles) both get a 2-way K split (two CTAs per tile fit the
# 148 SMs) with different split starts; 10000 rows (79 tiles) get none, the
# path that only clears the status word.
CASES = [(2000, 4096, 0.01, "topk", 24), (6000, 2048, 0.005, "zipf", 80), (10000, 1024, 0.01, "uniform", 16)]


def test_two_calls_in_a_row_match_dsq_gemv(orc):
    mats = []
    for i, (rows, cols, dens, kind, batch) in enumerate(CASES):
        p = synth.make_problem(rows, cols, 3, "affine", dens, kind, 900 + i, 1)
        blob = dsq.pack_problem(p)
        mats.append((p, blob, dsq.blob_desc(blob), upload(blob), dsq.Handle(blob), batch))
    calls = [(0, 11), (1, 12), (1, 13), (2, 15), (0, 14), (2, 16)]
    for m, seed in calls:
        p, blob, desc, dev_blob, h, batch = mats[m]
        xb = random_x(seed, batch, p.cols)
        x = to_dev(xb)
        y_new = torch.full((batch, p.rows), float("nan"), dtype=torch.float16, device="cuda")
        dsq.gemv_noalloc(desc, dev_blob, x, y_new)
        y_old = h.gemv(x)
        torch.cuda.synchronize()
        h.check()
        y_ref, bound = orc.gemv(p, x=xb)
        what = f"{p.rows}x{p.cols} B={batch} x-seed {seed}"
        within(to_f64(y_new), to_f64(y_old), bound, what)
        within(to_f64(y_new), y_ref, bound, what + " vs oracle")
    for *_, h, _ in mats:
        h.close()


def test_refusals():
    p = synth.make_problem(256, 512, 3, "affine", 0.01, "uniform", 5, 1)
    blob = dsq.pack_problem(p)
    desc = dsq.blob_desc(blob)
    dev_blob = upload(blob)
    x = torch.zeros((16, 512), dtype=torch.float16, device="cuda")
    y = torch.zeros((16, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(dsq.DSQError) as e:   # batch below the tensor-core path's 16
        dsq.gemv_noalloc(desc, dev_blob, x[:8].contiguous(), y[:8].contiguous())
    assert e.value.status == dsq.DSQ_ERR_UNSUPPORTED
    with pytest.raises(dsq.DSQError) as e:   # not the blob's size
        dsq.gemv_noalloc(desc, dev_blob[:-16], x, y)
    assert e.value.status == dsq.DSQ_ERR_INVALID_ARG
    q = synth.make_problem(256, 512, 4, "lut", 0.01, "uniform", 6, 1)
    qblob = dsq.pack_problem(q)
    with pytest.raises(dsq.DSQError) as e:   # LUT matrices are not covered
        dsq.gemv_noalloc(dsq.blob_desc(qblob), upload(qblob), x, y)
    assert e.value.status == dsq.DSQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
