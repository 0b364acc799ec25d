"""The oracle over a whole large input, on several host threads.

Test infrastructure. Rows (row-wise QDQ, STE) and columns (column-wise QDQ)
are independent, so the input is cut into disjoint row or column chunks and
each chunk goes through the oracle's own entry points unchanged; the chunk
results are placed side by side. ctypes releases the GIL for the duration of
each C call and the oracle keeps no state between calls, so the chunks run
in parallel on plain threads (no process pool, nothing forked after the GPU
is initialised). Column chunks are whole octets of columns wide, so packed
codes and mask bytes of a chunk are whole bytes of the full result.
"""
from __future__ import annotations

import concurrent.futures
import os

import numpy as np

import oracle as O


def threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _pool():
    return concurrent.futures.ThreadPoolExecutor(max_workers=threads())


def _row_chunks(rows: int, parts: int):
    step = max(1, -(-rows // parts))
    return [(r0, min(rows, r0 + step)) for r0 in range(0, rows, step)]


def _col_chunks(cols: int, parts: int):
    step = max(8, (-(-cols // parts) + 7) // 8 * 8)
    return [(c0, min(cols, c0 + step)) for c0 in range(0, cols, step)]


def _rowwise_into(fn, x: np.ndarray, out: dict, r0: int, r1: int, *args):
    part = fn(np.ascontiguousarray(x[r0:r1]), *args)
    for k, v in part.items():
        out[k][r0:r1] = v


def _colwise_into(fn, x: np.ndarray, out: dict, c0: int, c1: int, code_bytes_per_col: float, *args):
    part = fn(np.ascontiguousarray(x[:, c0:c1]), *args)
    out["y"][:, c0:c1] = part["y"]
    out["scales"][:, c0:c1] = part["scales"]
    out["codes"][:, int(c0 * code_bytes_per_col):int(c0 * code_bytes_per_col) + part["codes"].shape[1]] = part["codes"]
    out["mask"][:, c0 // 8:c0 // 8 + part["mask"].shape[1]] = part["mask"]


def _alloc(x: np.ndarray, code_cols: int, scale_rows: int, scale_cols: int) -> dict:
    rows, cols = x.shape
    return dict(y=np.empty_like(x), codes=np.zeros((rows, code_cols), np.uint8),
                scales=np.zeros((scale_rows, scale_cols), np.uint8),
                mask=np.zeros((rows, (cols + 7) // 8), np.uint8))


def qdq_rowwise(x: np.ndarray, block: int = 32, scale_factor: float = 6.0, mode: int = O.SCALE_PAGE) -> dict:
    """O.qdq_rowwise of the whole array, row chunks in parallel."""
    rows, cols = x.shape
    out = _alloc(x, (cols + 1) // 2, rows, (cols + block - 1) // block)
    with _pool() as p:
        fs = [p.submit(_rowwise_into, O.qdq_rowwise, x, out, r0, r1, block, scale_factor, mode)
              for r0, r1 in _row_chunks(rows, 4 * threads())]
        for f in fs:
            f.result()
    return out


def qdq_colwise(x: np.ndarray, block: int = 32, scale_factor: float = 6.0, mode: int = O.SCALE_PAGE,
                ends=None) -> dict:
    """O.qdq_colwise of the whole array, column chunks in parallel."""
    rows, cols = x.shape
    e = np.array([rows], np.int64) if ends is None else np.asarray(ends, np.int64)
    s = O.colwise_scale_rows(e, block)
    out = _alloc(x, (cols + 1) // 2, s, cols)
    with _pool() as p:
        fs = [p.submit(_colwise_into, O.qdq_colwise, x, out, c0, c1, 0.5, block, scale_factor, mode, ends)
              for c0, c1 in _col_chunks(cols, 4 * threads())]
        for f in fs:
            f.result()
    return out


def qdq8_rowwise(x: np.ndarray) -> dict:
    """O.qdq8_rowwise (MXFP8) of the whole array, row chunks in parallel."""
    rows, cols = x.shape
    out = _alloc(x, cols, rows, (cols + 31) // 32)
    with _pool() as p:
        fs = [p.submit(_rowwise_into, O.qdq8_rowwise, x, out, r0, r1) for r0, r1 in _row_chunks(rows, 4 * threads())]
        for f in fs:
            f.result()
    return out


def qdq8_colwise(x: np.ndarray, ends=None) -> dict:
    """O.qdq8_colwise (MXFP8) of the whole array, column chunks in parallel."""
    rows, cols = x.shape
    e = np.array([rows], np.int64) if ends is None else np.asarray(ends, np.int64)
    s = O.colwise_scale_rows(e, 32)
    out = _alloc(x, cols, s, cols)
    with _pool() as p:
        fs = [p.submit(_colwise_into, O.qdq8_colwise, x, out, c0, c1, 1.0, ends)
              for c0, c1 in _col_chunks(cols, 4 * threads())]
        for f in fs:
            f.result()
    return out


def ste_bwd(grad_out: np.ndarray, mask: np.ndarray, clip_grad: bool = True) -> np.ndarray:
    """O.ste_bwd of the whole array, row chunks in parallel."""
    rows = grad_out.shape[0]
    out = np.empty_like(grad_out)

    def one(r0, r1):
        out[r0:r1] = O.ste_bwd(np.ascontiguousarray(grad_out[r0:r1]), np.ascontiguousarray(mask[r0:r1]), clip_grad)

    with _pool() as p:
        fs = [p.submit(one, r0, r1) for r0, r1 in _row_chunks(rows, 4 * threads())]
        for f in fs:
            f.result()
    return out


def dual_level_rowwise(x: np.ndarray, level0_block: int = 512, scale_factor: float = 6.0,
                       mode: int = O.SCALE_PAGE) -> dict:
    """O.dual_level_rowwise of the whole array, row chunks in parallel."""
    rows, cols = x.shape
    out = dict(y=np.empty_like(x), codes=np.zeros((rows, (cols + 1) // 2), np.uint8),
               scales0=np.zeros((rows, -(-cols // level0_block)), np.float32),
               scales1=np.zeros((rows, -(-cols // 32)), np.uint8), mask=np.zeros((rows, (cols + 7) // 8), np.uint8))
    with _pool() as p:
        fs = [p.submit(_rowwise_into, O.dual_level_rowwise, x, out, r0, r1, level0_block, scale_factor, mode)
              for r0, r1 in _row_chunks(rows, 4 * threads())]
        for f in fs:
            f.result()
    return out
