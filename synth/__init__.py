"""Seeded synthetic workloads for the dense-and-sparse quantized GEMV.

This module only *produces inputs*: the logical dense codes with their
per-row lookup tables or per-group scale/zero pairs, the CSR outliers and the
fp16 activations.  It never decodes a weight and never forms a product, so it
holds none of the arithmetic that the oracle and the CUDA path compute; both
of them consume what it returns.

What the workloads imitate (all draws come from ``numpy.random.default_rng``):

* Base weights ``W ~ N(0, 0.02^2)`` in fp64, then Laplace(0, 0.2) spikes added
  at the chosen outlier positions (SpQR page, "Qu'est-ce qu'un poids outlier ?":
  a Gaussian bulk with a few very large weights).
* The outliers leave the dense part (they become holes, "trous") and go to a
  CSR store of fp16 values with column indices and row pointers (SpQR page,
  "Le format de stockage sparse"; SqueezeLLM page, "Dense-and-Sparse
  decomposition", W = W_dense + W_sparse).  The stored value is the original
  weight rounded to fp16.
* Dense part, one of two encodings:
  - ``lut``: SqueezeLLM-style non-uniform bins, one fp16 table of 2^bits
    centroids per output row (SqueezeLLM page, "Sensitivity-based
    non-uniform quantization").  The centroids are the row's odd quantiles
    (2k+1)/2^(bits+1) of its non-hole weights; each weight takes the nearest
    centroid (ties to the lower index), a hole takes the centroid nearest 0.
  - ``affine``: SpQR-style uniform codes over groups of 16 input columns
    (SpQR page, quant_config "wbits" and "groupsize": 16) with an fp16 scale
    and an integral fp16 zero per group; ``w ~ scale * (q - zero)``.  The range
    of a group is widened to contain 0 so that holes encode exactly.
* ``x ~ N(0, 1)`` rounded to fp16, drawn after everything else.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

LUT = "lut"
AFFINE = "affine"
BITPLANE = "bitplane"
INTGRID = "intgrid"
GROUP = 16
INTGRID_MAX = 8191


def bitplane_group(bits: int) -> int:
    """Inputs per coefficient group of a bit-plane matrix with `bits` planes."""
    return 32 << bits


def round_half_up(v: float) -> int:
    return int(math.floor(v + 0.5))


def f16_bits(a) -> np.ndarray:
    """fp64 values -> fp16 bit patterns (numpy's round-to-nearest-even)."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


@dataclasses.dataclass
class Problem:
    """One quantized layer plus activations, in logical (unpacked) form.

    codes   uint8  [rows, cols]          one code per weight, < 2^bits
    table   uint16 [rows, 2^bits]        lut: fp16 centroids of each row
            uint16 [rows, cols/16]       affine: fp16 scale of each group
    zeros   uint16 [rows, cols/16]       affine: fp16 integral zero; lut: None
    row_ptr int32  [rows+1]              CSR row pointers
    col_idx int32  [nnz]                 CSR column indices, increasing per row
    values  uint16 [nnz]                 CSR fp16 outlier values
    x       uint16 [batch, cols]         fp16 activations
    row_scale, col_scale  uint16 [rows] / [cols] fp16 two-axis scales, or None
    """
    name: str
    rows: int
    cols: int
    bits: int
    mode: str
    codes: np.ndarray
    table: np.ndarray
    zeros: Optional[np.ndarray]
    row_ptr: np.ndarray
    col_idx: np.ndarray
    values: np.ndarray
    x: np.ndarray
    row_scale: Optional[np.ndarray] = None
    col_scale: Optional[np.ndarray] = None

    @property
    def nnz(self) -> int:
        return int(self.row_ptr[-1])

    @property
    def batch(self) -> int:
        return int(self.x.shape[0])

    def with_x(self, x: np.ndarray) -> "Problem":
        return dataclasses.replace(self, x=np.ascontiguousarray(x, dtype=np.uint16))

    def canonical_bytes(self, batch: Optional[int] = None) -> int:
        """Bytes one product moves under the canonical accounting: packed
        codes, fp16 table or fp16 scale + fp16 zero, CSR as fp16 value +
        int32 column + int32 row pointer, fp16 x and y."""
        b = self.batch if batch is None else batch
        codes = self.rows * self.cols * self.bits // 8
        if self.mode == LUT:
            meta = self.rows * (1 << self.bits) * 2
        elif self.mode == BITPLANE:
            meta = self.rows * (self.cols // bitplane_group(self.bits)) * (self.bits + 1) * 2
        elif self.mode == INTGRID:
            # Huffman-coded integers: code bits, fp16 scales, slot bit offsets, codebook
            codes = (huffman_bits(self.codes) + 7) // 8
            nsym = int(np.unique(self.codes).size)
            meta = self.rows * (self.cols // GROUP) * 2 + self.rows * ((self.cols + 31) // 32) * 4 \
                + (65 + 1024) * 4 + 2 * nsym
        else:
            meta = self.rows * (self.cols // GROUP) * 4
        csr = self.nnz * 6 + (self.rows + 1) * 4
        if self.row_scale is not None:
            meta += (self.rows + self.cols) * 2
        return codes + meta + csr + b * self.cols * 2 + b * self.rows * 2


# ---------------------------------------------------------------- outliers

def _distinct_cells(rng, n_want: int, draw, taken: set) -> List[int]:
    """Draw flat cell indices with ``draw(k)`` until n_want new distinct ones
    (not already in ``taken``) are collected; collisions are redrawn."""
    out: List[int] = []
    while len(out) < n_want:
        cand = draw(max(2 * (n_want - len(out)), 16))
        for c in cand.tolist():
            if c not in taken:
                taken.add(c)
                out.append(c)
                if len(out) == n_want:
                    break
    return out


def _structured_positions(rng, M: int, N: int, nnz: int) -> np.ndarray:
    """Half of the outliers in 2% of rows and 2% of columns, half uniform."""
    rows_sel = rng.choice(M, math.ceil(0.02 * M), replace=False)
    cols_sel = rng.choice(N, math.ceil(0.02 * N), replace=False)
    n_struct = nnz // 2
    n_rowpart = n_struct // 2
    n_colpart = n_struct - n_rowpart
    n_uniform = nnz - n_struct
    taken: set = set()
    pos = _distinct_cells(
        rng, n_rowpart,
        lambda k: rows_sel[rng.integers(0, len(rows_sel), k)] * N + rng.integers(0, N, k),
        taken)
    pos += _distinct_cells(
        rng, n_colpart,
        lambda k: rng.integers(0, M, k) * N + cols_sel[rng.integers(0, len(cols_sel), k)],
        taken)
    pos += _distinct_cells(rng, n_uniform, lambda k: rng.integers(0, M * N, k), taken)
    return np.asarray(pos, dtype=np.int64)


def zipf_row_counts(rng, M: int, N: int, nnz: int, alpha: float = 1.2) -> np.ndarray:
    """Per-row outlier counts proportional to rank^-alpha for a seeded random
    ranking of the rows, summing to nnz, each clipped at N (the excess of a
    clipped row is spread over the unclipped rows; leftover units go to the
    largest fractional remainders)."""
    rank = np.empty(M, dtype=np.int64)
    rank[rng.permutation(M)] = np.arange(1, M + 1)
    w = rank.astype(np.float64) ** (-alpha)
    if nnz > M * N:
        raise ValueError("more outliers than cells")
    target = np.zeros(M, dtype=np.float64)
    clipped = np.zeros(M, dtype=bool)
    remaining = float(nnz)
    for _ in range(M + 1):
        free = ~clipped
        share = w[free] / w[free].sum() * remaining
        over = share > N
        if not over.any():
            target[free] = share
            break
        idx = np.flatnonzero(free)[over]
        target[idx] = N
        clipped[idx] = True
        remaining = nnz - target[clipped].sum()
    counts = np.floor(target).astype(np.int64)
    left = nnz - int(counts.sum())
    if left > 0:
        rem = target - counts
        rem[counts >= N] = -1.0
        order = np.argsort(-rem, kind="stable")
        counts[order[:left]] += 1
    assert counts.sum() == nnz and counts.max() <= N
    return counts


def _zipf_positions(rng, M: int, N: int, nnz: int) -> np.ndarray:
    counts = zipf_row_counts(rng, M, N, nnz)
    pos = []
    for r in range(M):
        if counts[r]:
            pos.append(r * N + np.sort(rng.choice(N, int(counts[r]), replace=False)))
    return np.concatenate(pos).astype(np.int64) if pos else np.zeros(0, np.int64)


# ---------------------------------------------------------------- dense part

def _quantize_lut(Wd: np.ndarray, hole: np.ndarray, bits: int):
    M, N = Wd.shape
    K = 1 << bits
    levels = (2.0 * np.arange(K) + 1.0) / (2.0 * K)
    table = np.zeros((M, K), dtype=np.uint16)
    codes = np.zeros((M, N), dtype=np.uint8)
    chunk = max(1, (1 << 22) // max(1, N * K))
    for r0 in range(0, M, chunk):
        r1 = min(M, r0 + chunk)
        cent = np.zeros((r1 - r0, K), dtype=np.float64)
        for r in range(r0, r1):
            vals = Wd[r][~hole[r]]
            if vals.size:
                cent[r - r0] = np.quantile(vals, levels)
        tb = f16_bits(cent)
        table[r0:r1] = tb
        c16 = tb.view(np.float16).astype(np.float64)
        w = np.where(hole[r0:r1], 0.0, Wd[r0:r1])
        dist = np.abs(w[:, :, None] - c16[:, None, :])
        codes[r0:r1] = np.argmin(dist, axis=2).astype(np.uint8)
    return codes, table


def _quantize_affine(Wd: np.ndarray, bits: int):
    M, N = Wd.shape
    qmax = (1 << bits) - 1
    G = Wd.reshape(M, N // GROUP, GROUP)
    mn = np.minimum(G.min(axis=2), 0.0)
    mx = np.maximum(G.max(axis=2), 0.0)
    s16 = f16_bits((mx - mn) / qmax)
    sval = s16.view(np.float16).astype(np.float64)
    degenerate = ~(np.isfinite(sval) & (sval > 0))
    sval = np.where(degenerate, 1.0, sval)
    s16 = np.where(degenerate, np.uint16(0x3C00), s16).astype(np.uint16)
    zero = np.clip(np.rint(-mn / sval), 0, qmax)
    zero = np.where(degenerate, 0.0, zero)
    q = np.rint(G / sval[:, :, None]) + zero[:, :, None]
    codes = np.clip(q, 0, qmax).astype(np.uint8).reshape(M, N)
    return codes, s16, f16_bits(zero)


def _quantize_bitplane(Wd: np.ndarray, hole: np.ndarray, bits: int):
    """Bit planes and per-group coefficients (BPDQ page, "Optimisation":
    planes from a bit-plane decomposition, coefficients by least squares).
    Without a Hessian the metric is the identity: each group's non-hole
    weights are rounded onto a uniform k-bit grid spanning their range (0
    included), the planes are that code's bits, and C0..Ck are the least-
    squares fit of the weights on [1, b_1, .., b_k], rounded to fp16."""
    M, N = Wd.shape
    K, G = 1 << bits, bitplane_group(bits)
    ng = N // G
    W3 = np.where(hole, 0.0, Wd).reshape(M, ng, G)
    keep = (~hole).reshape(M, ng, G)
    mn = np.minimum(np.where(keep, W3, np.inf).min(axis=2), 0.0)
    mx = np.maximum(np.where(keep, W3, -np.inf).max(axis=2), 0.0)
    step = (mx - mn) / (K - 1)
    step = np.where(step > 0, step, 1.0)
    q = np.clip(np.rint((W3 - mn[:, :, None]) / step[:, :, None]), 0, K - 1).astype(np.int64)
    planes = np.stack([(q >> i) & 1 for i in range(bits)], axis=3).astype(np.float64)  # M, ng, G, k
    A = np.concatenate([np.ones((M, ng, G, 1)), planes], axis=3) * keep[:, :, :, None]
    AtA = np.einsum("mgjp,mgjq->mgpq", A, A)
    Atw = np.einsum("mgjp,mgj->mgp", A, W3 * keep)
    coef = np.einsum("mgpq,mgq->mgp", np.linalg.pinv(AtA), Atw)
    return q.reshape(M, N).astype(np.uint8), f16_bits(coef)


def huffman_bits(q: np.ndarray) -> int:
    """Total length of an optimal Huffman code of the integers q (the
    canonical byte count of an integer-grid matrix)."""
    import heapq
    _, counts = np.unique(q, return_counts=True)
    if counts.size == 1:
        return int(counts[0])
    heap = [int(c) for c in counts]
    heapq.heapify(heap)
    total = 0
    while len(heap) > 1:
        a, b = heapq.heappop(heap), heapq.heappop(heap)
        total += a + b
        heapq.heappush(heap, a + b)
    return total


def _quantize_intgrid(W: np.ndarray):
    """One unconstrained integer grid per group of 16 (the HPTQ bullet): the
    step is half of a robust spread of the group (1.4826 * median |w|), so
    the Gaussian bulk spans a few levels and spikes land on large integers."""
    M, N = W.shape
    G = W.reshape(M, N // GROUP, GROUP)
    spread = 1.4826 * np.median(np.abs(G), axis=2)
    s16 = f16_bits(np.where(spread > 0, spread / 2.0, 1.0))
    sv = s16.view(np.float16).astype(np.float64)
    q = np.clip(np.rint(G / sv[:, :, None]), -INTGRID_MAX, INTGRID_MAX).astype(np.int16)
    return q.reshape(M, N), s16


# ---------------------------------------------------------------- assembly

def _two_axis_scales(Wd: np.ndarray, hole: np.ndarray, iters: int = 8):
    """Row and column scales that even out the spread of the dense weights
    (SINQ page, "Sinkhorn-Knopp": alternate normalisations of the rows' and
    the columns' standard deviations).  Returns the fp16 scales and the
    matrix divided by them."""
    keep = ~hole
    n_r = np.maximum(keep.sum(axis=1), 1)
    n_c = np.maximum(keep.sum(axis=0), 1)
    r = np.ones(Wd.shape[0])
    c = np.ones(Wd.shape[1])
    for _ in range(iters):
        A = np.where(keep, Wd / np.outer(r, c), 0.0)
        sr = np.sqrt((A * A).sum(axis=1) / n_r)
        r *= np.where(sr > 0, sr, 1.0)
        A = np.where(keep, Wd / np.outer(r, c), 0.0)
        sc = np.sqrt((A * A).sum(axis=0) / n_c)
        c *= np.where(sc > 0, sc, 1.0)
    r16, c16 = f16_bits(r), f16_bits(c)
    rv = r16.view(np.float16).astype(np.float64)
    cv = c16.view(np.float16).astype(np.float64)
    return r16, c16, np.where(hole, 0.0, Wd / np.outer(rv, cv))


def make_problem(rows: int, cols: int, bits: int, mode: str, density: float,
                 outliers: str = "uniform", seed: int = 0, batch: int = 1,
                 name: str = "", two_axis: bool = False) -> Problem:
    """Build one layer: outlier kind is 'topk', 'uniform', 'structured',
    'zipf' or 'none'.  two_axis: the weights carry log-normal row and column
    gains, and the dense part is quantized after dividing out two-axis
    scales, which the problem then holds."""
    if cols % GROUP:
        raise ValueError("cols must be a multiple of 16")
    M, N = rows, cols
    rng = np.random.default_rng(seed)
    W = rng.normal(0.0, 0.02, size=(M, N))
    if two_axis:
        W *= np.outer(np.exp(rng.normal(0.0, 0.5, M)), np.exp(rng.normal(0.0, 0.5, N)))
    nnz = round_half_up(density * M * N) if outliers != "none" else 0
    Wf = W.reshape(-1)
    if mode == INTGRID:
        # inliers and outliers share the grid: the spikes stay in the matrix
        if nnz:
            spike_pos = rng.choice(M * N, nnz, replace=False)
            Wf[spike_pos] += rng.laplace(0.0, 0.2, nnz)
        codes, table = _quantize_intgrid(W)
        x = f16_bits(rng.normal(0.0, 1.0, size=(batch, N)))
        return Problem(name=name, rows=M, cols=N, bits=14, mode=mode, codes=codes, table=table,
                       zeros=None, row_ptr=np.zeros(M + 1, np.int32), col_idx=np.zeros(0, np.int32),
                       values=np.zeros(0, np.uint16), x=x)
    if nnz == 0:
        pos = np.zeros(0, dtype=np.int64)
    elif outliers in ("topk", "uniform"):
        spike_pos = rng.choice(M * N, nnz, replace=False)
        Wf[spike_pos] += rng.laplace(0.0, 0.2, nnz)
        if outliers == "topk":
            pos = np.argsort(-np.abs(Wf), kind="stable")[:nnz]
        else:
            pos = spike_pos
    elif outliers == "structured":
        pos = _structured_positions(rng, M, N, nnz)
        Wf[pos] += rng.laplace(0.0, 0.2, nnz)
    elif outliers == "zipf":
        pos = _zipf_positions(rng, M, N, nnz)
        Wf[pos] += rng.laplace(0.0, 0.2, nnz)
    else:
        raise ValueError(outliers)
    pos = np.sort(np.asarray(pos, dtype=np.int64))
    values = f16_bits(Wf[pos])
    r_of = pos // N
    col_idx = (pos % N).astype(np.int32)
    row_ptr = np.zeros(M + 1, dtype=np.int32)
    np.add.at(row_ptr, r_of + 1, 1)
    row_ptr = np.cumsum(row_ptr).astype(np.int32)
    hole = np.zeros((M, N), dtype=bool)
    hole.reshape(-1)[pos] = True
    Wd = np.where(hole, 0.0, W)
    del W, Wf
    row_scale = col_scale = None
    if two_axis:
        row_scale, col_scale, Wd = _two_axis_scales(Wd, hole)
    if mode == LUT:
        codes, table = _quantize_lut(Wd, hole, bits)
        zeros = None
    elif mode == AFFINE:
        codes, table, zeros = _quantize_affine(Wd, bits)
    elif mode == BITPLANE:
        if cols % bitplane_group(bits):
            raise ValueError("bit-plane cols must be a multiple of 32 * 2^bits")
        codes, table = _quantize_bitplane(Wd, hole, bits)
        zeros = None
    else:
        raise ValueError(mode)
    x = f16_bits(rng.normal(0.0, 1.0, size=(batch, N)))
    return Problem(name=name, rows=M, cols=N, bits=bits, mode=mode, codes=codes,
                   table=table, zeros=zeros, row_ptr=row_ptr, col_idx=col_idx,
                   values=values, x=x, row_scale=row_scale, col_scale=col_scale)


# ---------------------------------------------------------------- raw weights

def spiky_weights(rows: int, cols: int, density: float, seed: int) -> np.ndarray:
    """Unquantized fp32 weights shaped like the workloads' (N(0, 0.02^2) plus
    Laplace(0, 0.2) spikes at round(density * rows * cols) uniform positions),
    the input of the on-device decomposition."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.02, size=(rows, cols))
    n = round_half_up(density * rows * cols)
    pos = rng.choice(rows * cols, n, replace=False)
    w.reshape(-1)[pos] += rng.laplace(0.0, 0.2, n)
    return w.astype(np.float32)


# ---------------------------------------------------------------- the five workloads

C4_LAYERS = (("q", 6656, 6656), ("k", 6656, 6656), ("v", 6656, 6656),
             ("o", 6656, 6656), ("gate", 17920, 6656), ("up", 17920, 6656),
             ("down", 6656, 17920))

CONFIGS: Dict[str, dict] = {
    "c0": dict(rows=1024, cols=1024, bits=3, mode=LUT, density=0.01,
               outliers="topk", seed=0, batches=(1,),
               about="1024x1024 3-bit row-LUT, 1% top-|w| outliers after Laplace spikes"),
    "c1": dict(rows=4096, cols=4096, bits=3, mode=LUT, density=0.0045,
               outliers="uniform", seed=1, batches=(1,),
               about="4096x4096 3-bit row-LUT, 0.45% uniform outliers"),
    "c2": dict(rows=11008, cols=4096, bits=3, mode=AFFINE, density=0.01,
               outliers="structured", seed=2, batches=(1,),
               about="11008x4096 3-bit affine g16, 1% structured outliers"),
    "c3": dict(rows=4096, cols=11008, bits=4, mode=LUT, density=0.005,
               outliers="zipf", seed=3, batches=(1, 2, 4, 8),
               about="4096x11008 4-bit row-LUT, 0.5% Zipf(1.2) row-skewed outliers"),
    # BPDQ variable-grid matrices on the 11008x4096 shape of c2
    "bp2": dict(rows=11008, cols=4096, bits=2, mode=BITPLANE, density=0.01,
                outliers="uniform", seed=52, batches=(1, 2, 4),
                about="11008x4096 2-bit-plane BPDQ (groups of 128, 3 fp16 coefficients), 1% uniform outliers"),
    "bp3": dict(rows=11008, cols=4096, bits=3, mode=BITPLANE, density=0.01,
                outliers="uniform", seed=53, batches=(1, 2, 4),
                about="11008x4096 3-bit-plane BPDQ (groups of 256, 4 fp16 coefficients), 1% uniform outliers"),
    # Huffman-coded integer grid (HPTQ), inliers and spikes on one grid, same shape
    "hq": dict(rows=11008, cols=4096, bits=14, mode=INTGRID, density=0.01,
               outliers="uniform", seed=70, batches=(1, 2),
               about="11008x4096 Huffman-coded integer grid (HPTQ), fp16 scale per 16, 1% Laplace spikes in the grid"),
    # SINQ two-axis scales around a non-uniform 3-bit table, same shape
    "sq3": dict(rows=11008, cols=4096, bits=3, mode=LUT, density=0.01,
                outliers="uniform", seed=60, batches=(1, 2), two_axis=True,
                about="11008x4096 3-bit row-LUT with SINQ two-axis fp16 scales, 1% uniform outliers"),
}


def config_names() -> List[str]:
    return ["c0", "c1", "c2", "c3"] + ["c4_" + n for n, _, _ in C4_LAYERS]


def make_config(name: str, batch: Optional[int] = None) -> Problem:
    """Workload by name: c0..c3, or c4_<layer> for the seven linear layers of
    the 6656-hidden / 17920-FFN block.  The activations hold the largest batch
    of the config's sweep (8 for c3, 16 for c4) unless ``batch`` is given;
    smaller batches take the leading rows."""
    if name.startswith("c4_"):
        layer = name[3:]
        for li, (ln, M, N) in enumerate(C4_LAYERS):
            if ln == layer:
                return make_problem(M, N, 3, AFFINE, 0.01, "uniform", 40 + li,
                                    16 if batch is None else batch, name)
        raise KeyError(name)
    c = CONFIGS[name]
    b = max(c["batches"]) if batch is None else batch
    return make_problem(c["rows"], c["cols"], c["bits"], c["mode"], c["density"],
                        c["outliers"], c["seed"], b, name, c.get("two_axis", False))


def describe(name: str) -> str:
    if name.startswith("c4_"):
        for ln, M, N in C4_LAYERS:
            if "c4_" + ln == name:
                return f"{M}x{N} 3-bit affine g16, 1% uniform outliers ({ln} of the 33B-scale block)"
    return CONFIGS[name]["about"]
