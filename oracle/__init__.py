"""ctypes front of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg use it; the CUDA library never does.  ``load()`` compiles
``oracle.c`` with gcc into ``liboracle.so`` beside it when that is missing or
older than the source, or takes another source file (tests compile planted
mistakes that way, into a temporary directory).

Each function takes a problem object with the attributes ``rows, cols, bits,
mode ('lut' | 'affine' | 'bitplane'), codes, table, zeros, row_ptr, col_idx,
values`` as
numpy arrays of the dtypes the synthetic generator produces.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64


def compile_library(source: str = SOURCE, output: str = LIBRARY) -> str:
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", output,
                    source, "-lm"], check=True)
    return output


def _needs_build(source: str, output: str) -> bool:
    return (not os.path.exists(output)
            or os.path.getmtime(output) < os.path.getmtime(source))


class Oracle:
    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_double_to_half.restype = ctypes.c_uint16
        lib.oracle_double_to_half.argtypes = [ctypes.c_double]
        lib.oracle_half_to_double_n.argtypes = [_P, _P, _I64]
        lib.oracle_double_to_half_n.argtypes = [_P, _P, _I64]
        lib.oracle_decode.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P]
        lib.oracle_materialize.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_gemv_rows.restype = _I
        lib.oracle_gemv_rows.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I,
                                         _P, _P, _I, _P, _P]
        lib.oracle_decompose.restype = _I
        lib.oracle_decompose.argtypes = [_I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_materialize_two_axis.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                                    _P, _P, _P]
        lib.oracle_gemv_rows_two_axis.restype = _I
        lib.oracle_gemv_rows_two_axis.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                                  _P, _P, _I, _P, _P, _I, _P, _P]
        self.lib = lib
        self.path = path

    # -- fp16 <-> fp64 -------------------------------------------------
    def half_to_double(self, h) -> np.ndarray:
        h = np.ascontiguousarray(h, dtype=np.uint16)
        out = np.empty(h.shape, dtype=np.float64)
        self.lib.oracle_half_to_double_n(h.ctypes.data, out.ctypes.data, h.size)
        return out

    def double_to_half(self, v) -> np.ndarray:
        v = np.ascontiguousarray(v, dtype=np.float64)
        out = np.empty(v.shape, dtype=np.uint16)
        self.lib.oracle_double_to_half_n(v.ctypes.data, out.ctypes.data, v.size)
        return out

    # -- the method ----------------------------------------------------
    @staticmethod
    def _args(p):
        mode = {"lut": 0, "affine": 1, "bitplane": 2, "intgrid": 3}[p.mode]
        codes = np.ascontiguousarray(p.codes, dtype=np.int16 if mode == 3 else np.uint8)
        table = np.ascontiguousarray(p.table, dtype=np.uint16)
        zeros = (np.ascontiguousarray(p.zeros, dtype=np.uint16)
                 if p.zeros is not None else None)
        rp = np.ascontiguousarray(p.row_ptr, dtype=np.int32)
        ci = np.ascontiguousarray(p.col_idx, dtype=np.int32)
        va = np.ascontiguousarray(p.values, dtype=np.uint16)
        rs = getattr(p, "row_scale", None)
        cs = getattr(p, "col_scale", None)
        rs = None if rs is None else np.ascontiguousarray(rs, dtype=np.uint16)
        cs = None if cs is None else np.ascontiguousarray(cs, dtype=np.uint16)
        keep = (codes, table, zeros, rp, ci, va, rs, cs)
        ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
        return keep, (int(p.rows), int(p.cols), int(p.bits), mode, ptr(codes),
                      ptr(table), ptr(zeros), ptr(rp), ptr(ci), ptr(va)), (ptr(rs), ptr(cs))

    def decode(self, p) -> np.ndarray:
        """W_dense as fp16 bit patterns, rows x cols."""
        keep, a, _ = self._args(p)
        out = np.empty((p.rows, p.cols), dtype=np.uint16)
        self.lib.oracle_decode(*a[:7], out.ctypes.data)
        return out

    def materialize(self, p) -> np.ndarray:
        """What = W_dense + W_sparse in fp64, rows x cols (the dense part
        times r_i * c_j when the problem carries row_scale / col_scale)."""
        keep, a, sc = self._args(p)
        out = np.empty((p.rows, p.cols), dtype=np.float64)
        self.lib.oracle_materialize_two_axis(*a, *sc, out.ctypes.data)
        return out

    def gemv(self, p, x: Optional[np.ndarray] = None,
             rows: Optional[Sequence[int]] = None):
        """(y_ref, bound), each batch x len(rows) fp64; all rows by default."""
        keep, a, sc = self._args(p)
        x = np.ascontiguousarray(p.x if x is None else x, dtype=np.uint16)
        if x.ndim == 1:
            x = x[None, :]
        batch = x.shape[0]
        if rows is None:
            rl, n = None, int(p.rows)
        else:
            rl = np.ascontiguousarray(rows, dtype=np.int32)
            n = int(rl.size)
        y = np.empty((batch, n), dtype=np.float64)
        bound = np.empty((batch, n), dtype=np.float64)
        rc = self.lib.oracle_gemv_rows_two_axis(*a, *sc, batch, x.ctypes.data,
                                                None if rl is None else rl.ctypes.data, n,
                                                y.ctypes.data, bound.ctypes.data)
        if rc != 0:
            raise MemoryError("oracle_gemv_rows failed")
        return y, bound


    # -- the decomposition before the product -------------------------
    def decompose(self, w: np.ndarray, bits: int, mode: str, nnz: int):
        """Outliers (the nnz largest |w|) and the quantized dense part of fp32
        weights w [rows, cols]: (codes, table, zeros, row_ptr, col_idx,
        values) as dsq_pack takes them."""
        w = np.ascontiguousarray(w, dtype=np.float32)
        rows, cols = w.shape
        m = {"lut": 0, "affine": 1}[mode]
        codes = np.empty((rows, cols), np.uint8)
        if m == 0:
            table, zeros = np.empty((rows, 1 << bits), np.uint16), None
        else:
            table, zeros = np.empty((rows, cols // 16), np.uint16), np.empty((rows, cols // 16), np.uint16)
        rp = np.empty(rows + 1, np.int32)
        ci = np.empty(max(nnz, 1), np.int32)
        va = np.empty(max(nnz, 1), np.uint16)
        rc = self.lib.oracle_decompose(rows, cols, bits, m, nnz, w.ctypes.data, codes.ctypes.data,
                                       table.ctypes.data, None if zeros is None else zeros.ctypes.data,
                                       rp.ctypes.data, ci.ctypes.data, va.ctypes.data)
        if rc != 0:
            raise MemoryError("oracle_decompose failed")
        return codes, table, zeros, rp, ci[:nnz], va[:nnz]


_default: Optional[Oracle] = None


def load(source: str = SOURCE, output: Optional[str] = None) -> Oracle:
    """The oracle library built from ``source`` (compiled when stale)."""
    global _default
    if source == SOURCE and output is None:
        if _default is None:
            if _needs_build(SOURCE, LIBRARY):
                compile_library(SOURCE, LIBRARY)
            _default = Oracle(LIBRARY)
        return _default
    out = output or os.path.splitext(source)[0] + ".so"
    compile_library(source, out)
    return Oracle(out)
