"""Python binding of libdsq (the dense-and-sparse quantized GEMV for B200).

Argument marshalling only: every step of the product runs in the library's
CUDA kernels.  PyTorch supplies device memory and streams.  The binding
refuses to work without the compiled library (``python -m
dense_sparse_quantized_b200.build``); there is no fallback path.

    blob = pack(rows, cols, bits, mode, codes, table, zeros, row_ptr, col_idx, values)
    h = Handle(blob, device=0)
    y = h.gemv(x)              # x: cuda fp16 [batch, cols] -> y: cuda fp16 [batch, rows]
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(HERE, "libdsq.so")

DSQ_OK = 0
DSQ_ERR_INVALID_ARG = -1
DSQ_ERR_UNSUPPORTED = -2
DSQ_ERR_CUDA = -3
DSQ_ERR_OOM = -4
DSQ_ERR_BUFFER_TOO_SMALL = -5
DSQ_ERR_DEVICE = -6
DSQ_ERR_SCRATCH_LIMIT = -7
MODE_LUT_ROW = 0
MODE_AFFINE_G16 = 1
MODE_BITPLANE = 2
MODE_INTGRID = 3

EXPORTS = ("dsq_pack", "dsq_pack_two_axis", "dsq_pack_intgrid", "dsq_blob_desc", "dsq_create", "dsq_gemv", "dsq_gemv_launches", "dsq_decode",
           "dsq_handle_desc", "dsq_device_bytes", "dsq_check", "dsq_destroy", "dsq_status_string",
           "dsq_gemv_noalloc", "dsq_selftest_wait_timeout", "dsq_decompose")


class DSQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class Desc(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int32), ("cols", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("nnz", ctypes.c_int64)]


_lib = None


def library() -> ctypes.CDLL:
    """The loaded libdsq.so; raises when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY):
            raise RuntimeError(f"{LIBRARY} is missing: build it with "
                               "`python -m dense_sparse_quantized_b200.build`")
        lib = ctypes.CDLL(LIBRARY)
        P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.dsq_pack.argtypes = [ctypes.POINTER(Desc), P, P, P, P, P, P, P, ctypes.POINTER(SZ)]
        lib.dsq_pack_two_axis.argtypes = [ctypes.POINTER(Desc), P, P, P, P, P, P, P, P, P,
                                          ctypes.POINTER(SZ)]
        lib.dsq_pack_intgrid.argtypes = [ctypes.POINTER(Desc), P, P, P, P, P, P, ctypes.POINTER(SZ)]
        lib.dsq_blob_desc.argtypes = [P, SZ, ctypes.POINTER(Desc)]
        lib.dsq_create.argtypes = [P, SZ, I, ctypes.POINTER(P)]
        lib.dsq_gemv.argtypes = [P, P, P, I, P]
        lib.dsq_gemv_launches.argtypes = [P, I]
        lib.dsq_decode.argtypes = [P, P, P]
        lib.dsq_handle_desc.argtypes = [P, ctypes.POINTER(Desc)]
        lib.dsq_device_bytes.argtypes = [P]
        lib.dsq_device_bytes.restype = SZ
        lib.dsq_check.argtypes = [P]
        lib.dsq_destroy.argtypes = [P]
        lib.dsq_gemv_noalloc.argtypes = [ctypes.POINTER(Desc), P, SZ, P, P, I, P]
        lib.dsq_selftest_wait_timeout.argtypes = [P, P]
        lib.dsq_decompose.argtypes = [ctypes.POINTER(Desc), P, P, P, P, P, P, P, P, ctypes.POINTER(SZ), P]
        lib.dsq_status_string.argtypes = [I]
        lib.dsq_status_string.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name != "dsq_status_string" and name != "dsq_device_bytes":
                getattr(lib, name).restype = I
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().dsq_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != DSQ_OK:
        raise DSQError(rc, what)


def _arr(a, dtype):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def pack(rows: int, cols: int, bits: int, mode, codes, table, zeros, row_ptr, col_idx,
         values, row_scale=None, col_scale=None) -> bytes:
    """Validate logical weights and return the packed blob (host bytes).

    mode: 'lut' / 'affine' / 'bitplane' or MODE_*.  Arrays: codes uint8
    [rows, cols]; table fp16 bits (uint16) [rows, 2^bits] (lut),
    [rows, cols/16] (affine scales) or [rows, cols/(32*2^bits), bits+1]
    (bit-plane coefficients C0..Ck); zeros uint16 [rows, cols/16] or None;
    row_ptr int32; col_idx int32; values uint16 fp16 bits.  row_scale /
    col_scale (fp16 bits [rows] / [cols]): two-axis scales (dsq_pack_two_axis)."""
    lib = library()
    m = {"lut": MODE_LUT_ROW, "affine": MODE_AFFINE_G16, "bitplane": MODE_BITPLANE}.get(mode, mode)
    nnz = int(np.asarray(row_ptr)[-1]) if row_ptr is not None and len(row_ptr) else 0
    d = Desc(int(rows), int(cols), int(bits), int(m), nnz)
    keep = [_arr(codes, np.uint8), _arr(table, np.uint16), _arr(zeros, np.uint16),
            _arr(row_ptr, np.int32), _arr(col_idx, np.int32), _arr(values, np.uint16)]
    two = row_scale is not None or col_scale is not None
    if two:
        keep += [_arr(row_scale, np.uint16), _arr(col_scale, np.uint16)]
    ptrs = [p for _, p in keep]
    fn, name = (lib.dsq_pack_two_axis, "dsq_pack_two_axis") if two else (lib.dsq_pack, "dsq_pack")
    size = ctypes.c_size_t(0)
    rc = fn(ctypes.byref(d), *ptrs, None, ctypes.byref(size))
    if rc != DSQ_ERR_BUFFER_TOO_SMALL:
        _check(rc, name)
    buf = ctypes.create_string_buffer(size.value)
    _check(fn(ctypes.byref(d), *ptrs, buf, ctypes.byref(size)), name)
    return buf.raw[:size.value]


def pack_intgrid(rows: int, cols: int, q, scales, row_ptr, col_idx, values) -> bytes:
    """Huffman-code an integer-grid matrix (dsq_pack_intgrid): q int16
    [rows, cols] (|q| <= 8191), scales fp16 bits [rows, cols/16], optional
    outliers as CSR."""
    lib = library()
    nnz = int(np.asarray(row_ptr)[-1]) if row_ptr is not None and len(row_ptr) else 0
    d = Desc(int(rows), int(cols), 14, MODE_INTGRID, nnz)
    keep = [_arr(q, np.int16), _arr(scales, np.uint16), _arr(row_ptr, np.int32),
            _arr(col_idx, np.int32), _arr(values, np.uint16)]
    ptrs = [p for _, p in keep]
    size = ctypes.c_size_t(0)
    rc = lib.dsq_pack_intgrid(ctypes.byref(d), *ptrs, None, ctypes.byref(size))
    if rc != DSQ_ERR_BUFFER_TOO_SMALL:
        _check(rc, "dsq_pack_intgrid")
    buf = ctypes.create_string_buffer(size.value)
    _check(lib.dsq_pack_intgrid(ctypes.byref(d), *ptrs, buf, ctypes.byref(size)), "dsq_pack_intgrid")
    return buf.raw[:size.value]


def pack_problem(p) -> bytes:
    """pack() from an object with rows, cols, bits, mode, codes, table, zeros,
    row_ptr, col_idx, values attributes."""
    if p.mode == "intgrid":
        return pack_intgrid(p.rows, p.cols, p.codes, p.table, p.row_ptr, p.col_idx, p.values)
    return pack(p.rows, p.cols, p.bits, p.mode, p.codes, p.table, p.zeros, p.row_ptr,
                p.col_idx, p.values, getattr(p, "row_scale", None), getattr(p, "col_scale", None))


def blob_desc(blob: bytes) -> Desc:
    d = Desc()
    _check(library().dsq_blob_desc(blob, len(blob), ctypes.byref(d)), "dsq_blob_desc")
    return d


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


class Handle:
    """A packed matrix resident on one GPU."""

    def __init__(self, blob: bytes, device: int = 0):
        self._h = None
        h = ctypes.c_void_p()
        _check(library().dsq_create(blob, len(blob), int(device), ctypes.byref(h)), "dsq_create")
        self._h = h
        self.device = int(device)
        d = Desc()
        _check(library().dsq_handle_desc(h, ctypes.byref(d)), "dsq_handle_desc")
        self.rows, self.cols, self.bits, self.mode, self.nnz = d.rows, d.cols, d.bits, d.mode, d.nnz

    @property
    def device_bytes(self) -> int:
        return int(library().dsq_device_bytes(self._h))

    def gemv(self, x, y=None, stream=None):
        """y = x @ What^T.  x: cuda fp16 [batch, cols] (or [cols]); y optional
        cuda fp16 [batch, rows].  Asynchronous on ``stream`` (default: the
        current torch stream)."""
        import torch
        squeeze = x.dim() == 1
        if squeeze:
            x = x.unsqueeze(0)
        if x.dtype != torch.float16 or not x.is_cuda or not x.is_contiguous():
            raise ValueError("x must be a contiguous cuda float16 tensor")
        if x.shape[1] != self.cols:
            raise ValueError(f"x has {x.shape[1]} columns, the matrix {self.cols}")
        batch = x.shape[0]
        if y is None:
            y = torch.empty((batch, self.rows), dtype=torch.float16, device=x.device)
        elif (y.dtype != torch.float16 or not y.is_cuda or not y.is_contiguous()
              or tuple(y.shape) != (batch, self.rows)):
            raise ValueError("y must be a contiguous cuda float16 tensor [batch, rows]")
        _check(library().dsq_gemv(self._h, x.data_ptr(), y.data_ptr(), batch,
                                  _stream_ptr(stream)), "dsq_gemv")
        return y[0] if squeeze else y

    def launches_per_call(self, batch: int) -> int:
        """Kernel launches one gemv() of this batch makes."""
        n = library().dsq_gemv_launches(self._h, int(batch))
        if n < 0:
            raise DSQError(DSQ_ERR_INVALID_ARG, "dsq_gemv_launches")
        return n

    def gemv_host(self, x_host, y_host=None, x_dev=None, y_dev=None, stream=None):
        """End-to-end call from host memory: copy x (pinned cpu fp16
        [batch, cols]) to the device, run the product, copy y back into pinned
        cpu memory.  Asynchronous; synchronise the stream before reading y."""
        import torch
        if x_dev is None:
            x_dev = torch.empty(x_host.shape, dtype=torch.float16, device=f"cuda:{self.device}")
        if y_host is None:
            y_host = torch.empty((x_host.shape[0], self.rows), dtype=torch.float16).pin_memory()
        if y_dev is None:
            y_dev = torch.empty(y_host.shape, dtype=torch.float16, device=x_dev.device)
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            x_dev.copy_(x_host, non_blocking=True)
            self.gemv(x_dev, y_dev, stream=s)
            y_host.copy_(y_dev, non_blocking=True)
        return y_host

    def decode(self, out=None, stream=None):
        """W_dense as cuda fp16 [rows, cols] (outliers not added)."""
        import torch
        if out is None:
            out = torch.empty((self.rows, self.cols), dtype=torch.float16,
                              device=f"cuda:{self.device}")
        _check(library().dsq_decode(self._h, out.data_ptr(), _stream_ptr(stream)), "dsq_decode")
        return out

    def check(self):
        """Synchronise the device; raise if a kernel of this handle gave up a
        bounded wait since the last check."""
        _check(library().dsq_check(self._h), "dsq_check")

    def selftest_wait_timeout(self, stream=None):
        """Test hook: launch a kernel whose bounded wait runs out (about 2 s);
        the next check() raises DSQ_ERR_DEVICE."""
        _check(library().dsq_selftest_wait_timeout(self._h, _stream_ptr(stream)),
               "dsq_selftest_wait_timeout")

    def close(self):
        if self._h is not None:
            _check(library().dsq_destroy(self._h), "dsq_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def gemv_noalloc(desc: Desc, packed_device, x, y, stream=None):
    """y = x @ What^T without a handle and without any device allocation in
    the library, for callers whose device memory all comes from a host
    program's own pool.  ``packed_device``: the dsq_pack blob already copied
    to the device by the caller (a cuda uint8 tensor, 256-byte aligned);
    ``x``: cuda fp16 [batch, cols]; ``y``: caller-allocated cuda fp16
    [batch, rows].  Calls that overlap on the GPU share one scratch array and
    race.  Asynchronous on ``stream`` (default: the current torch stream)."""
    import torch
    if packed_device.dtype != torch.uint8 or not packed_device.is_cuda or not packed_device.is_contiguous():
        raise ValueError("packed_device must be a contiguous cuda uint8 tensor")
    for name, t in (("x", x), ("y", y)):
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 2:
            raise ValueError(f"{name} must be a contiguous 2-D cuda float16 tensor")
    batch = x.shape[0]
    if x.shape[1] != desc.cols or tuple(y.shape) != (batch, desc.rows):
        raise ValueError("x must be [batch, cols] and y [batch, rows]")
    _check(library().dsq_gemv_noalloc(ctypes.byref(desc), packed_device.data_ptr(), packed_device.numel(),
                                      x.data_ptr(), y.data_ptr(), batch, _stream_ptr(stream)),
           "dsq_gemv_noalloc")
    return y


def decompose(w, bits: int, mode: str, nnz: int, stream=None, workspace=None):
    """Outliers and quantized dense part of device fp32 weights w [rows, cols]
    (dsq_decompose): returns cuda tensors (codes, table, zeros or None,
    row_ptr, col_idx, values) -- the arrays pack() takes.  ``workspace``:
    an optional cuda uint8 tensor to reuse; one is allocated otherwise."""
    import torch
    if w.dtype != torch.float32 or not w.is_cuda or not w.is_contiguous() or w.dim() != 2:
        raise ValueError("w must be a contiguous 2-D cuda float32 tensor")
    rows, cols = w.shape
    m = {"lut": MODE_LUT_ROW, "affine": MODE_AFFINE_G16}[mode]
    d = Desc(rows, cols, int(bits), m, int(nnz))
    dev = w.device
    size = ctypes.c_size_t(0)
    rc = library().dsq_decompose(ctypes.byref(d), None, None, None, None, None, None, None, None,
                                 ctypes.byref(size), None)
    if rc != DSQ_ERR_BUFFER_TOO_SMALL:
        _check(rc, "dsq_decompose")
    if workspace is None or workspace.numel() < size.value:
        workspace = torch.empty(max(size.value, 1), dtype=torch.uint8, device=dev)
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    if m == MODE_LUT_ROW:
        table = torch.empty((rows, 1 << bits), dtype=torch.float16, device=dev)
        zeros = None
    else:
        table = torch.empty((rows, cols // 16), dtype=torch.float16, device=dev)
        zeros = torch.empty((rows, cols // 16), dtype=torch.float16, device=dev)
    row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
    values = torch.empty(max(nnz, 1), dtype=torch.float16, device=dev)
    size = ctypes.c_size_t(workspace.numel())
    _check(library().dsq_decompose(ctypes.byref(d), w.data_ptr(), codes.data_ptr(), table.data_ptr(),
                                   None if zeros is None else zeros.data_ptr(), row_ptr.data_ptr(),
                                   col_idx.data_ptr(), values.data_ptr(), workspace.data_ptr(),
                                   ctypes.byref(size), _stream_ptr(stream)), "dsq_decompose")
    return codes, table, zeros, row_ptr, col_idx[:nnz], values[:nnz]
