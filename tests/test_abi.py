"""Host-side checks of the C ABI: the library loads, exports what include/*.h
declares, validates inputs with the documented status codes, and lays out the
blob as layout.h describes.  No GPU and no kernel launch."""
import ctypes
import glob
import os
import re
import subprocess
import types

import numpy as np
import pytest

import dense_sparse_quantized_b200 as dsq
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        for m in re.finditer(r"^DSQ_API\s+[\w\s\*]+?\b(dsq_\w+)\s*\(", open(h).read(), re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert {"dsq_pack", "dsq_create", "dsq_gemv", "dsq_decode", "dsq_destroy",
            "dsq_status_string"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", dsq.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dsq_\w+)", out))
    assert names <= exported, names - exported
    lib = dsq.library()
    for n in names:
        assert hasattr(lib, n)


def test_status_strings():
    for s in (0, -1, -2, -3, -4, -5, -6, 99):
        assert isinstance(dsq.status_string(s), str) and dsq.status_string(s)


def test_null_handle_calls_are_rejected_on_the_host():
    lib = dsq.library()
    assert lib.dsq_gemv(None, None, None, 1, None) == dsq.DSQ_ERR_INVALID_ARG
    assert lib.dsq_decode(None, None, None) == dsq.DSQ_ERR_INVALID_ARG
    assert lib.dsq_destroy(None) == dsq.DSQ_OK
    assert lib.dsq_device_bytes(None) == 0
    assert lib.dsq_create(None, 0, 0, None) == dsq.DSQ_ERR_INVALID_ARG
    assert lib.dsq_selftest_wait_timeout(None, None) == dsq.DSQ_ERR_INVALID_ARG


# --------------------------------------------------------------- validation

def small(bits=3, mode="affine", rows=5, cols=48, seed=0, density=0.05):
    return synth.make_problem(rows, cols, bits, mode, density, "uniform", seed, 1)


def pack_status(p, **over):
    a = dict(rows=p.rows, cols=p.cols, bits=p.bits, mode=p.mode, codes=p.codes,
             table=p.table, zeros=p.zeros, row_ptr=p.row_ptr, col_idx=p.col_idx,
             values=p.values)
    a.update(over)
    try:
        dsq.pack(**a)
        return dsq.DSQ_OK
    except dsq.DSQError as e:
        return e.status


def test_pack_accepts_valid_inputs():
    for bits in (3, 4):
        for mode in ("lut", "affine"):
            assert pack_status(small(bits, mode)) == dsq.DSQ_OK


@pytest.mark.parametrize("case", [
    "bits2", "bits5", "cols_not16", "bad_mode", "code_too_big", "zeros_for_lut",
    "no_zeros_affine", "zero_not_integral", "zero_too_big", "scale_nan", "scale_overflow",
    "table_inf", "rowptr_start", "rowptr_end", "rowptr_decreasing", "col_unsorted",
    "col_duplicate", "col_out_of_range", "col_negative", "value_nan", "null_codes"])
def test_pack_rejects(case):
    p = small(3, "affine")
    pl = small(3, "lut")
    bad = dict(
        bits2=(p, dict(bits=2)), bits5=(p, dict(bits=5)),
        cols_not16=(p, dict(cols=40)), bad_mode=(p, dict(mode=7)),
        code_too_big=(p, dict(codes=np.where(np.arange(p.codes.size).reshape(p.codes.shape) == 7, 8, p.codes))),
        zeros_for_lut=(pl, dict(zeros=np.zeros((5, 3), np.uint16))),
        no_zeros_affine=(p, dict(zeros=None)),
        zero_not_integral=(p, dict(zeros=np.full_like(p.zeros, 0x3800))),   # 0.5
        zero_too_big=(p, dict(zeros=np.full_like(p.zeros, 0x4800))),        # 8
        scale_nan=(p, dict(table=np.full_like(p.table, 0x7E00))),
        scale_overflow=(p, dict(table=np.full_like(p.table, 0x7400))),      # 16384 * max(z, 7-z) >= 65536
        table_inf=(pl, dict(table=np.full_like(pl.table, 0x7C00))),
        rowptr_start=(p, dict(row_ptr=p.row_ptr + 1)),
        rowptr_end=(p, dict(row_ptr=np.concatenate([p.row_ptr[:-1], [p.row_ptr[-1] + 1]]))),
        rowptr_decreasing=(p, dict(row_ptr=np.array([0, 3, 2, 5, 5, p.row_ptr[-1]]))),
        col_unsorted=(p, dict(col_idx=p.col_idx[::-1].copy())),
        col_duplicate=(p, dict(col_idx=np.where(np.arange(p.nnz) == 1, p.col_idx[0], p.col_idx))),
        col_out_of_range=(p, dict(col_idx=np.where(np.arange(p.nnz) == p.nnz - 1, 48, p.col_idx))),
        col_negative=(p, dict(col_idx=np.where(np.arange(p.nnz) == 0, -1, p.col_idx))),
        value_nan=(p, dict(values=np.full_like(p.values, 0x7E00))),
        null_codes=(p, dict(codes=None)),
    )[case]
    assert pack_status(bad[0], **bad[1]) == dsq.DSQ_ERR_INVALID_ARG


def test_pack_unsupported_width():
    lib = dsq.library()
    d = dsq.Desc(1, 65536, 3, 1, 0)
    size = ctypes.c_size_t(0)
    assert lib.dsq_pack(ctypes.byref(d), None, None, None, None, None, None, None,
                        ctypes.byref(size)) == dsq.DSQ_ERR_UNSUPPORTED


def test_pack_size_query_and_small_buffer():
    p = small()
    lib = dsq.library()
    d = dsq.Desc(p.rows, p.cols, p.bits, 1, p.nnz)
    arrs = [np.ascontiguousarray(a) for a in (p.codes, p.table, p.zeros)] + \
           [np.ascontiguousarray(p.row_ptr, np.int32), np.ascontiguousarray(p.col_idx, np.int32),
            np.ascontiguousarray(p.values)]
    size = ctypes.c_size_t(0)
    rc = lib.dsq_pack(ctypes.byref(d), *[a.ctypes.data for a in arrs], None, ctypes.byref(size))
    assert rc == dsq.DSQ_ERR_BUFFER_TOO_SMALL and size.value > 0
    need = size.value
    buf = ctypes.create_string_buffer(need)
    size = ctypes.c_size_t(need - 1)
    rc = lib.dsq_pack(ctypes.byref(d), *[a.ctypes.data for a in arrs], buf, ctypes.byref(size))
    assert rc == dsq.DSQ_ERR_BUFFER_TOO_SMALL and size.value == need


def test_blob_desc_and_corruption():
    p = small(4, "lut")
    blob = dsq.pack_problem(p)
    d = dsq.blob_desc(blob)
    assert (d.rows, d.cols, d.bits, d.mode, d.nnz) == (5, 48, 4, 0, p.nnz)
    bad = bytearray(blob)
    bad[0] ^= 0xFF
    with pytest.raises(dsq.DSQError):
        dsq.blob_desc(bytes(bad))
    with pytest.raises(dsq.DSQError):
        dsq.blob_desc(blob[:100])


def test_empty_shapes_pack():
    for rows, cols in ((0, 16), (3, 0), (0, 0)):
        blob = dsq.pack(rows, cols, 3, "affine", np.zeros((rows, cols), np.uint8),
                        np.zeros((rows, cols // 16), np.uint16), np.zeros((rows, cols // 16), np.uint16),
                        np.zeros(rows + 1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.uint16))
        d = dsq.blob_desc(blob)
        assert (d.rows, d.cols, d.nnz) == (rows, cols, 0)


# --------------------------------------------------------------- layout round trip

def unpack_blob(blob: bytes):
    """Test-only reader of the blob, written from the layout description:
    returns codes, table/scales, zeros, row_ptr, col_idx, values."""
    rows, cols, bits, mode = np.frombuffer(blob[16:32], np.int32)
    nnz = int(np.frombuffer(blob[32:40], np.int64)[0])
    S, row_words = np.frombuffer(blob[40:48], np.int32)
    off_dense, off_table, off_rp, off_csr, reserved0, total = np.frombuffer(blob[48:96], np.uint64)
    rec = np.frombuffer(blob[int(off_dense):int(off_dense) + rows * row_words * 4],
                        np.uint32).reshape(rows, row_words)

    def place(c, k):
        if bits == 4:
            return c // 8, 4 * (c % 8) + k
        if bits == 2:
            return c // 16, 2 * (c % 16) + k
        if c < 30:
            t = c % 10
            return c // 10, (16 if t % 2 else 0) + [0, 3, 6, 10, 13][t // 2] + k
        return k, (9 if c == 30 else 25)

    def word_of(s, p_):
        # word index inside a record of code word p_ (3 = scale pair) of slot s
        if (bits == 3 and mode == 0) or mode == 2:
            return p_ * S + s
        if bits == 3:
            return 136 * (s // 32) + 8 + 4 * (s % 32) + p_
        return 4 * s + p_ if p_ < 4 else 4 * S + s

    def zero_byte(s):
        return 4 * 136 * (s // 32) + s % 32 if bits == 3 else 4 * 5 * S + s

    codes = np.zeros((rows, cols), np.uint8)
    for s in range(S):
        words = [rec[:, word_of(s, p_)] for p_ in range(bits)]
        for c in range(32):
            j = 32 * s + c
            if j >= cols:
                break
            q = np.zeros(rows, np.uint32)
            for k in range(bits):
                wi, pos = place(c, k)
                q |= ((words[wi] >> np.uint32(pos)) & np.uint32(1)) << np.uint32(k)
            codes[:, j] = q
    G = cols // 16
    if mode == 0:
        table = np.frombuffer(blob[int(off_table):int(off_table) + rows * (1 << bits) * 2],
                              np.uint16).reshape(rows, 1 << bits)
        zeros = None
    elif mode == 2:   # level tables: 2^bits levels of each group, rows x S
        table = np.frombuffer(blob[int(off_table):int(off_table) + rows * S * 2],
                              np.uint16).reshape(rows, S)
        zeros = None
    else:
        table = np.zeros((rows, G), np.uint16)
        zeros = np.zeros((rows, G), np.uint16)
        for s in range(S):
            pair = rec[:, word_of(s, 3) if bits == 3 else 4 * S + s]
            zb = rec.view(np.uint8)[:, zero_byte(s)]
            for e in range(2):
                g = 2 * s + e
                if g < G:
                    table[:, g] = (pair >> np.uint32(16 * e)) & np.uint32(0xFFFF)
                    zeros[:, g] = np.asarray((zb >> (4 * e)) & 15, np.float64).astype(np.float16).view(np.uint16)
    row_ptr = np.frombuffer(blob[int(off_rp):int(off_rp) + (rows + 1) * 4], np.int32)
    csr = np.frombuffer(blob[int(off_csr):int(off_csr) + nnz * 4], np.uint32)
    col = (csr & np.uint32(0xFFFF)).astype(np.int32)
    val = (csr >> np.uint32(16)).astype(np.uint16)
    assert reserved0 == 0 and int(off_csr) + nnz * 4 + 12 <= total
    assert total == len(blob)
    return codes, table, zeros, row_ptr, col, val


@pytest.mark.parametrize("bits,mode,cols", [(3, "lut", 48), (4, "lut", 80), (3, "affine", 48),
                                            (4, "affine", 112), (3, "affine", 1024), (3, "lut", 16),
                                            (3, "affine", 1040), (3, "affine", 2048 + 512 + 16)])
def test_layout_round_trip(bits, mode, cols):
    p = synth.make_problem(7, cols, bits, mode, 0.03, "uniform", 2, 1)
    codes, table, zeros, rp, ci, va = unpack_blob(dsq.pack_problem(p))
    assert np.array_equal(codes, p.codes)
    assert np.array_equal(table, p.table)
    if mode == "affine":
        assert np.array_equal(zeros, p.zeros)
    assert np.array_equal(rp, p.row_ptr) and np.array_equal(ci, p.col_idx)
    assert np.array_equal(va, p.values)


@pytest.mark.parametrize("bits,cols", [(2, 128), (2, 1024), (3, 256), (3, 4096)])
def test_bitplane_layout_and_levels(orc, bits, cols):
    """Bit-plane blobs: the codes round-trip, and the level table holds, for
    every group g and code q, the oracle's decoded weight of a column of
    group g whose code is q."""
    p = synth.make_problem(9, cols, bits, "bitplane", 0.03, "uniform", 3 + bits, 1)
    codes, levels, zeros, rp, ci, va = unpack_blob(dsq.pack_problem(p))
    assert zeros is None and np.array_equal(codes, p.codes)
    assert np.array_equal(rp, p.row_ptr) and np.array_equal(ci, p.col_idx) and np.array_equal(va, p.values)
    K, G = 1 << bits, synth.bitplane_group(bits)
    probe = types.SimpleNamespace(**vars(p))
    probe.codes = np.tile(np.arange(cols) % K, (p.rows, 1)).astype(np.uint8)
    wd = orc.decode(probe)
    want = np.stack([wd[:, g * G:g * G + K] for g in range(cols // G)], axis=1).reshape(p.rows, -1)
    assert np.array_equal(levels, want)


def test_bitplane_levels_round_once(orc):
    """Coefficients over every binade (subnormals, ties, sums past the fp16
    range excluded): the packed levels equal the oracle's single rounding of
    the exact sum."""
    rng = np.random.default_rng(17)
    for bits in (2, 3):
        K, G = 1 << bits, synth.bitplane_group(bits)
        rows, cols = 64, 4 * G
        e = rng.integers(-24, 12, size=(rows, cols // G, bits + 1)).astype(np.float64)
        v = rng.integers(1, 2048, size=e.shape) * np.exp2(e - 10) * rng.choice([-1.0, 1.0], e.shape)
        coef = np.asarray(v, np.float64).astype(np.float16).view(np.uint16)
        codes = np.tile(np.arange(cols) % K, (rows, 1)).astype(np.uint8)
        p = types.SimpleNamespace(rows=rows, cols=cols, bits=bits, mode="bitplane", codes=codes,
                                  table=coef, zeros=None, row_ptr=np.zeros(rows + 1, np.int32),
                                  col_idx=np.zeros(0, np.int32), values=np.zeros(0, np.uint16),
                                  x=np.zeros((1, cols), np.uint16))
        _, levels, _, _, _, _ = unpack_blob(dsq.pack_problem(p))
        wd = orc.decode(p)
        want = np.stack([wd[:, g * G:g * G + K] for g in range(cols // G)], axis=1).reshape(rows, -1)
        assert np.array_equal(levels, want), bits


def test_bitplane_pack_rejects():
    pb = synth.make_problem(4, 256, 2, "bitplane", 0.02, "uniform", 1, 1)
    assert pack_status(pb) == dsq.DSQ_OK
    assert pack_status(pb, bits=4) == dsq.DSQ_ERR_INVALID_ARG                  # 2 or 3 planes
    assert pack_status(pb, cols=192, codes=pb.codes[:, :192]) == dsq.DSQ_ERR_INVALID_ARG  # groups of 128
    assert pack_status(pb, zeros=np.zeros((4, 16), np.uint16)) == dsq.DSQ_ERR_INVALID_ARG
    assert pack_status(pb, table=np.full_like(pb.table, 0x7E00)) == dsq.DSQ_ERR_INVALID_ARG   # NaN
    big = pb.table.copy()
    big[1, 0] = [0x7BFF, 0x7BFF, 0x0000]       # level C0 + C1 = 131008 is past fp16
    assert pack_status(pb, table=big) == dsq.DSQ_ERR_INVALID_ARG


def test_two_axis_blob_sections_and_checks():
    """Two-axis blobs carry the row and column scales in their own sections,
    flagged in the header; bad scales are refused; a plain blob reader of
    the same shape (the no-allocation entry point) refuses the larger blob
    before touching a device."""
    p = synth.make_problem(9, 256, 3, "lut", 0.03, "uniform", 4, 1, two_axis=True)
    blob = dsq.pack_problem(p)
    plain = dsq.pack(p.rows, p.cols, p.bits, p.mode, p.codes, p.table, p.zeros, p.row_ptr, p.col_idx, p.values)
    assert len(blob) > len(plain)
    off_rs, off_cs = (int(v) for v in np.frombuffer(blob[96:112], np.uint64))
    flags = int(np.frombuffer(blob[112:116], np.uint32)[0])
    assert flags == 1 and int(np.frombuffer(plain[112:116], np.uint32)[0]) == 0
    assert np.array_equal(np.frombuffer(blob[off_rs:off_rs + 2 * p.rows], np.uint16), p.row_scale)
    assert np.array_equal(np.frombuffer(blob[off_cs:off_cs + 2 * p.cols], np.uint16), p.col_scale)
    codes, table, _, rp, ci, va = unpack_blob(blob)
    assert np.array_equal(codes, p.codes) and np.array_equal(table, p.table)
    d = dsq.blob_desc(blob)
    assert (d.rows, d.cols, d.bits, d.mode) == (9, 256, 3, 0)
    bad = bytearray(blob)
    bad[112:116] = np.array([2], np.uint32).tobytes()     # an unknown flag
    with pytest.raises(dsq.DSQError):
        dsq.blob_desc(bytes(bad))
    for rs, cs in ((np.full(9, 0x7E00, np.uint16), p.col_scale), (p.row_scale, np.full(256, 0x7C00, np.uint16))):
        with pytest.raises(dsq.DSQError) as e:
            dsq.pack(p.rows, p.cols, p.bits, p.mode, p.codes, p.table, p.zeros, p.row_ptr, p.col_idx,
                     p.values, rs, cs)
        assert e.value.status == dsq.DSQ_ERR_INVALID_ARG
    lib = dsq.library()
    desc = dsq.Desc(p.rows, p.cols, p.bits, dsq.MODE_LUT_ROW, p.nnz)
    assert lib.dsq_gemv_noalloc(ctypes.byref(desc), 256, len(blob), 16, 16, 16, None) == dsq.DSQ_ERR_INVALID_ARG


def decode_intgrid_blob(blob: bytes):
    """Test-only reader of an INTGRID blob, written from the format
    description: canonical code from the codebook's per-length counts, the
    MSB-first bitstream read code by code from each slot's bit offset."""
    rows, cols, bits, mode = (int(v) for v in np.frombuffer(blob[16:32], np.int32))
    S = int(np.frombuffer(blob[40:44], np.int32)[0])
    off_dense, off_table = (int(v) for v in np.frombuffer(blob[48:64], np.uint64))
    off_index, off_codebook = (int(v) for v in np.frombuffer(blob[120:136], np.uint64))
    stream_words, nsym = (int(v) for v in np.frombuffer(blob[136:144], np.uint32))
    cb = np.frombuffer(blob[off_codebook:off_codebook + 4 * (65 + 1024 + (nsym + 1) // 2)], np.uint32)
    assert cb[0] == nsym
    count = cb[23:44]
    syms = np.frombuffer(cb[65 + 1024:].tobytes()[:2 * nsym], np.int16)
    table = {}
    code, r = 0, 0
    for length in range(1, 21):                  # canonical: by length, then value
        for _ in range(int(count[length])):
            table[(length, code)] = int(syms[r])
            code += 1
            r += 1
        code <<= 1
    stream = np.frombuffer(blob[off_dense:off_dense + 4 * (stream_words + 24)], np.uint32)
    bitstr = np.unpackbits(stream.byteswap().view(np.uint8))   # MSB-first bit order
    idx = np.frombuffer(blob[off_index:off_index + 4 * rows * S], np.uint32).reshape(rows, S)
    q = np.zeros((rows, cols), np.int16)
    for i in range(rows):
        for s in range(S):
            pos = int(idx[i, s])
            for c in range(min(32, cols - 32 * s)):
                code, length = 0, 0
                while (length, code) not in table:
                    code = (code << 1) | int(bitstr[pos])
                    pos += 1
                    length += 1
                    assert length <= 20
                q[i, 32 * s + c] = table[(length, code)]
    scales = np.frombuffer(blob[off_table:off_table + 2 * rows * (cols // 16)], np.uint16).reshape(rows, -1)
    return q, scales


@pytest.mark.parametrize("rows,cols,seed", [(9, 256, 1), (3, 48, 2), (17, 1040, 3)])
def test_intgrid_blob_round_trip(rows, cols, seed):
    p = synth.make_problem(rows, cols, 14, "intgrid", 0.02, "uniform", seed, 1)
    q, scales = decode_intgrid_blob(dsq.pack_problem(p))
    assert np.array_equal(q, p.codes) and np.array_equal(scales, p.table)


def test_intgrid_long_codes_and_one_symbol():
    """Skewed frequencies force codes past the 10-bit fast table (and past 20
    bits before limiting); a matrix of one integer has a one-symbol code."""
    rng = np.random.default_rng(8)
    q = np.zeros((4, 4096), np.int16)
    q.reshape(-1)[:] = np.minimum(rng.geometric(0.5, q.size) - 1, 40).astype(np.int16) * np.where(rng.random(q.size) < 0.5, -1, 1)
    q[2, 5] = 8191
    q[3, 7] = -8191
    sc = np.full((4, 256), 0x3C00, np.uint16)
    blob = dsq.pack_intgrid(4, 4096, q, sc, np.zeros(5, np.int32), np.zeros(0, np.int32), np.zeros(0, np.uint16))
    assert np.array_equal(decode_intgrid_blob(blob)[0], q)
    nsym = int(np.frombuffer(blob[140:144], np.uint32)[0])
    off_cb = int(np.frombuffer(blob[128:136], np.uint64)[0])
    max_len = int(np.frombuffer(blob[off_cb + 4:off_cb + 8], np.uint32)[0])
    assert nsym > 20 and 10 < max_len <= 20          # codes past the fast table, limited to 20 bits
    one = np.full((2, 64), -3, np.int16)
    blob = dsq.pack_intgrid(2, 64, one, np.full((2, 4), 0x3C00, np.uint16), np.zeros(3, np.int32),
                            np.zeros(0, np.int32), np.zeros(0, np.uint16))
    assert np.array_equal(decode_intgrid_blob(blob)[0], one)


def test_intgrid_refusals():
    lib = dsq.library()
    q = np.zeros((2, 32), np.int16)
    sc = np.full((2, 2), 0x3C00, np.uint16)
    rp = np.zeros(3, np.int32)
    with pytest.raises(dsq.DSQError):
        dsq.pack_intgrid(2, 32, np.full((2, 32), 8192, np.int16), sc, rp, np.zeros(0, np.int32), np.zeros(0, np.uint16))
    with pytest.raises(dsq.DSQError):
        dsq.pack_intgrid(2, 32, q, np.full((2, 2), 0x7C00, np.uint16), rp, np.zeros(0, np.int32), np.zeros(0, np.uint16))
    size = ctypes.c_size_t(0)
    d = dsq.Desc(2, 32, 13, dsq.MODE_INTGRID, 0)           # bits must be 14
    assert lib.dsq_pack_intgrid(ctypes.byref(d), q.ctypes.data, sc.ctypes.data, rp.ctypes.data, None, None,
                                None, ctypes.byref(size)) == dsq.DSQ_ERR_INVALID_ARG
    d = dsq.Desc(2, 32, 14, dsq.MODE_INTGRID, 0)           # integers go through dsq_pack_intgrid only
    assert lib.dsq_pack(ctypes.byref(d), q.ctypes.data, sc.ctypes.data, None, rp.ctypes.data, None, None,
                        None, ctypes.byref(size)) == dsq.DSQ_ERR_INVALID_ARG
    blob = bytearray(dsq.pack_intgrid(2, 32, q, sc, rp, np.zeros(0, np.int32), np.zeros(0, np.uint16)))
    off_index = int(np.frombuffer(bytes(blob[120:128]), np.uint64)[0])
    blob[off_index:off_index + 4] = np.array([1 << 30], np.uint32).tobytes()   # a slot past the stream
    assert _create_rc(bytes(blob)) == dsq.DSQ_ERR_INVALID_ARG


def test_three_bit_fields():
    """3-bit placement: columns 2j and 2j+1 of a word's ten sit 16 bits apart
    (one mask puts both into the two 16-bit halves); every pair lies in bits
    0..9 of its halves, either in the word or in the word >> 10, so an AND
    alone makes two exact fp16 subnormals; columns 30/31 fill bits 9/25; the
    96 bits are used once each."""
    place = {}
    for c in range(32):
        for k in range(3):
            if c < 30:
                t = c % 10
                place[c, k] = (c // 10, (16 if t % 2 else 0) + [0, 3, 6, 10, 13][t // 2] + k)
            else:
                place[c, k] = (k, 9 if c == 30 else 25)
    assert len(set(place.values())) == 96
    for c in range(0, 30, 2):
        (w0, p0), (w1, p1) = place[c, 0], place[c + 1, 0]
        assert w0 == w1 and p1 == p0 + 16
        assert p0 + 2 <= 9 or (p0 >= 10 and p0 - 10 + 2 <= 9)


# --------------------------------------------------------------- blob contents at create

def _create_rc(blob: bytes) -> int:
    """dsq_create's status for a blob; a handle made where a GPU is present is freed.
    Without a device a blob that passes validation ends in DSQ_ERR_CUDA."""
    lib = dsq.library()
    h = ctypes.c_void_p()
    rc = lib.dsq_create(blob, len(blob), 0, ctypes.byref(h))
    if rc == dsq.DSQ_OK:
        lib.dsq_destroy(h)
    return rc


def _offsets(blob: bytes):
    rows = int(np.frombuffer(blob[16:20], np.int32)[0])
    off_rp, off_csr = (int(v) for v in np.frombuffer(blob[64:80], np.uint64))
    return rows, off_rp, off_csr


@pytest.mark.parametrize("bits,mode", [(3, "lut"), (4, "lut"), (3, "affine"), (4, "affine"),
                                       (2, "bitplane"), (3, "bitplane")])
def test_create_accepts_packed_blobs(bits, mode):
    shapes = ((7, 48, 0.05), (33, 1024, 0.02), (5, 16, 0.0), (1, 4096, 0.01))
    if mode == "bitplane":
        shapes = ((7, 256, 0.05), (33, 1024, 0.02), (5, 256, 0.0), (1, 4096, 0.01))
    for rows, cols, dens in shapes:
        p = synth.make_problem(rows, cols, bits, mode, dens, "uniform" if dens else "none", 9, 1)
        assert _create_rc(dsq.pack_problem(p)) in (dsq.DSQ_OK, dsq.DSQ_ERR_CUDA), (rows, cols, dens)


def test_create_rejects_corrupted_csr():
    """A blob whose row pointers or CSR columns would send a kernel outside
    its buffers is refused before any device work."""
    p = synth.make_problem(6, 64, 3, "affine", 0.1, "uniform", 4, 1)
    blob = dsq.pack_problem(p)
    assert _create_rc(blob) in (dsq.DSQ_OK, dsq.DSQ_ERR_CUDA)
    rows, off_rp, off_csr = _offsets(blob)
    rp = np.frombuffer(blob[off_rp:off_rp + 4 * (rows + 1)], np.int32).copy()
    busy = int(np.argmax(np.diff(rp)))  # a row with at least two entries
    assert rp[busy + 1] - rp[busy] >= 2

    def with_rp(new_rp):
        b = bytearray(blob)
        b[off_rp:off_rp + 4 * (rows + 1)] = np.asarray(new_rp, np.int32).tobytes()
        return bytes(b)

    def with_entry(k, col):
        b = bytearray(blob)
        e = int(np.frombuffer(blob[off_csr + 4 * k:off_csr + 4 * k + 4], np.uint32)[0])
        b[off_csr + 4 * k:off_csr + 4 * k + 4] = np.uint32((e & 0xFFFF0000) | col).tobytes()
        return bytes(b)

    bad = rp.copy(); bad[0] = 1
    assert _create_rc(with_rp(bad)) == dsq.DSQ_ERR_INVALID_ARG          # does not start at 0
    bad = rp.copy(); bad[-1] -= 1
    assert _create_rc(with_rp(bad)) == dsq.DSQ_ERR_INVALID_ARG          # does not end at nnz
    bad = rp.copy(); bad[busy + 1] = bad[busy] - 1 if bad[busy] > 0 else -1
    assert _create_rc(with_rp(bad)) == dsq.DSQ_ERR_INVALID_ARG          # decreasing
    k = int(rp[busy])
    assert _create_rc(with_entry(k, p.cols)) == dsq.DSQ_ERR_INVALID_ARG  # column out of range
    c_next = int(np.frombuffer(blob[off_csr + 4 * (k + 1):off_csr + 4 * (k + 2)], np.uint32)[0]) & 0xFFFF
    assert _create_rc(with_entry(k, c_next)) == dsq.DSQ_ERR_INVALID_ARG  # repeated column in a row
