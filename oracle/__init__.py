"""numpy bindings of the scalar CPU oracle (mxfp4_oracle.c).

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg import this package. The CUDA library and its binding never do.

mma_scale_layout restates the scale-factor layout of block-scaled tensor-core
GEMMs as the cuBLAS documentation defines it; the pages fix no such layout
(parity against them unpinned), and the tests pin it to hand-computed offsets
and to a derivation by reshapes.

bf16 data is passed as numpy uint16 arrays holding the raw bf16 bit patterns;
fp32 data as numpy float32 arrays. All arrays are 2-D [rows, cols] row-major.
"""
from __future__ import annotations

import ctypes

import numpy as np

from .build import LIB, build

F32, BF16 = 0, 1
SCALE_PAGE, SCALE_FLOOR = 0, 1

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = f32
        L.oracle_f32_to_bf16.argtypes = [f32]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_scale_page.argtypes = [f32, f32]
        L.oracle_scale_page.restype = f32
        L.oracle_scale_floor.argtypes = [f32]
        L.oracle_scale_floor.restype = f32
        L.oracle_qdq_block.argtypes = [P, i32, f32, i32, P, P, P, P]
        L.oracle_qdq_block.restype = None
        L.oracle_group_ends.argtypes = [P, i64, i32, i64, P]
        L.oracle_group_ends.restype = i32
        L.oracle_colwise_scale_rows.argtypes = [P, i64, i64]
        L.oracle_colwise_scale_rows.restype = i64
        L.oracle_qdq_rowwise.argtypes = [P, i32, i64, i64, i64, i32, f32, i32, P, P, P, P]
        L.oracle_qdq_rowwise.restype = i32
        L.oracle_qdq_colwise.argtypes = [P, i32, i64, i64, i64, i32, f32, i32, P, i64, P, P, P, P]
        L.oracle_qdq_colwise.restype = i32
        L.oracle_ste_bwd.argtypes = [P, i32, i64, i64, P, i32, P]
        L.oracle_ste_bwd.restype = None
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_qdq8_rowwise.argtypes = [P, i32, i64, i64, i64, P, P, P, P]
        L.oracle_qdq8_rowwise.restype = i32
        L.oracle_qdq8_colwise.argtypes = [P, i32, i64, i64, i64, P, i64, P, P, P, P]
        L.oracle_qdq8_colwise.restype = i32
        L.oracle_dual_level_rowwise.argtypes = [P, i64, i64, i64, i32, f32, i32, P, P, P, P, P]
        L.oracle_dual_level_rowwise.restype = i32
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return F32
    raise TypeError(f"oracle takes uint16 (bf16 bits) or float32, got {x.dtype}")


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f: float) -> int:
    return int(lib().oracle_f32_to_bf16(float(f)))


def scale_page(amax: float, scale_factor: float = 6.0) -> float:
    return float(lib().oracle_scale_page(amax, scale_factor))


def scale_floor(amax: float) -> float:
    return float(lib().oracle_scale_floor(amax))


def qdq_block(v, scale_factor: float = 6.0, mode: int = SCALE_PAGE):
    """One block of fp32 values -> (out f32[n], nibble u8[n], sat u8[n], e8m0 byte)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    n = v.size
    out = np.empty(n, np.float32)
    nib = np.empty(n, np.uint8)
    sat = np.empty(n, np.uint8)
    e8 = np.zeros(1, np.uint8)
    lib().oracle_qdq_block(_ptr(v), n, scale_factor, mode, _ptr(out), _ptr(nib), _ptr(sat), _ptr(e8))
    return out, nib, sat, int(e8[0])


def group_ends(group_list, group_list_type: int, rows: int) -> np.ndarray | None:
    """Cumulative end offsets of a group_list, or None when it is not a valid partition."""
    gl = np.ascontiguousarray(group_list, dtype=np.int64)
    ends = np.empty(max(gl.size, 1), np.int64)
    rc = lib().oracle_group_ends(_ptr(gl), gl.size, group_list_type, rows, _ptr(ends))
    return None if rc != 0 else ends[: gl.size]


def colwise_scale_rows(ends, block: int) -> int:
    e = np.ascontiguousarray(ends, dtype=np.int64)
    return int(lib().oracle_colwise_scale_rows(_ptr(e), e.size, block))


def qdq_rowwise(x: np.ndarray, block: int = 32, scale_factor: float = 6.0, mode: int = SCALE_PAGE):
    """Row-wise QDQ of a 2-D array; returns dict(y, codes, scales, mask)."""
    x = np.ascontiguousarray(x)
    dt = _dtype_code(x)
    rows, cols = x.shape
    y = np.empty_like(x)
    codes = np.zeros((rows, (cols + 1) // 2), np.uint8)
    scales = np.zeros((rows, (cols + block - 1) // block), np.uint8)
    mask = np.zeros((rows, (cols + 7) // 8), np.uint8)
    rc = lib().oracle_qdq_rowwise(_ptr(x), dt, rows, cols, cols, block, scale_factor, mode,
                                  _ptr(y), _ptr(codes), _ptr(scales), _ptr(mask))
    if rc != 0:
        raise MemoryError("oracle_qdq_rowwise failed")
    return dict(y=y, codes=codes, scales=scales, mask=mask)


def qdq_colwise(x: np.ndarray, block: int = 32, scale_factor: float = 6.0, mode: int = SCALE_PAGE,
                ends=None):
    """Column-wise QDQ (blocks down columns, restarting at group ends)."""
    x = np.ascontiguousarray(x)
    dt = _dtype_code(x)
    rows, cols = x.shape
    e = None if ends is None else np.ascontiguousarray(ends, dtype=np.int64)
    s = colwise_scale_rows(e if e is not None else np.array([rows], np.int64), block)
    y = np.empty_like(x)
    codes = np.zeros((rows, (cols + 1) // 2), np.uint8)
    scales = np.zeros((s, cols), np.uint8)
    mask = np.zeros((rows, (cols + 7) // 8), np.uint8)
    rc = lib().oracle_qdq_colwise(_ptr(x), dt, rows, cols, cols, block, scale_factor, mode,
                                  _ptr(e), 0 if e is None else e.size,
                                  _ptr(y), _ptr(codes), _ptr(scales), _ptr(mask))
    if rc != 0:
        raise MemoryError("oracle_qdq_colwise failed")
    return dict(y=y, codes=codes, scales=scales, mask=mask)


def qdq8_rowwise(x: np.ndarray):
    """Row-wise MXFP8 QDQ (E4M3 elements, E8M0 scale per 32): dict(y, codes
    [rows, cols] bytes, scales [rows, ceil(cols/32)], mask)."""
    x = np.ascontiguousarray(x)
    dt = _dtype_code(x)
    rows, cols = x.shape
    y = np.empty_like(x)
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((rows, (cols + 31) // 32), np.uint8)
    mask = np.zeros((rows, (cols + 7) // 8), np.uint8)
    lib().oracle_qdq8_rowwise(_ptr(x), dt, rows, cols, cols, _ptr(y), _ptr(codes), _ptr(scales), _ptr(mask))
    return dict(y=y, codes=codes, scales=scales, mask=mask)


def qdq8_colwise(x: np.ndarray, ends=None):
    """Column-wise MXFP8 QDQ (blocks of 32 rows restarting at group ends)."""
    x = np.ascontiguousarray(x)
    dt = _dtype_code(x)
    rows, cols = x.shape
    e = None if ends is None else np.ascontiguousarray(ends, dtype=np.int64)
    s = colwise_scale_rows(e if e is not None else np.array([rows], np.int64), 32)
    y = np.empty_like(x)
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((s, cols), np.uint8)
    mask = np.zeros((rows, (cols + 7) // 8), np.uint8)
    lib().oracle_qdq8_colwise(_ptr(x), dt, rows, cols, cols, _ptr(e), 0 if e is None else e.size,
                              _ptr(y), _ptr(codes), _ptr(scales), _ptr(mask))
    return dict(y=y, codes=codes, scales=scales, mask=mask)


def dual_level_rowwise(x: np.ndarray, level0_block: int = 512, scale_factor: float = 6.0,
                       mode: int = SCALE_PAGE):
    """Dual-level MX quantisation of bf16 bits [rows, cols] along rows:
    dict(y bf16 bits, codes [rows, ceil(cols/2)], scales0 fp32 [rows,
    ceil(cols/level0_block)], scales1 E8M0 [rows, ceil(cols/32)], mask)."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("dual-level quantisation takes bf16 bits (uint16)")
    rows, cols = x.shape
    y = np.empty_like(x)
    codes = np.zeros((rows, (cols + 1) // 2), np.uint8)
    s0 = np.zeros((rows, -(-cols // level0_block)), np.float32)
    s1 = np.zeros((rows, -(-cols // 32)), np.uint8)
    mask = np.zeros((rows, (cols + 7) // 8), np.uint8)
    rc = lib().oracle_dual_level_rowwise(_ptr(x), rows, cols, cols, level0_block, scale_factor, mode,
                                         _ptr(y), _ptr(codes), _ptr(s0), _ptr(s1), _ptr(mask))
    if rc != 0:
        raise ValueError("oracle_dual_level_rowwise: level0_block must be a positive multiple of 32")
    return dict(y=y, codes=codes, scales0=s0, scales1=s1, mask=mask)


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(code & 0x7F)) * (-1.0 if code & 0x80 else 1.0)


def e4m3_encode(y: float) -> int:
    return int(lib().oracle_e4m3_encode(y))


def ste_bwd(grad_out: np.ndarray, mask: np.ndarray, clip_grad: bool = True) -> np.ndarray:
    g = np.ascontiguousarray(grad_out)
    dt = _dtype_code(g)
    rows, cols = g.shape
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    assert m.shape == (rows, (cols + 7) // 8)
    out = np.empty_like(g)
    lib().oracle_ste_bwd(_ptr(g), dt, rows, cols, _ptr(m), int(bool(clip_grad)), _ptr(out))
    return out


def unpack_bits(mask: np.ndarray, cols: int) -> np.ndarray:
    """Bit-packed [rows, ceil(cols/8)] mask -> bool [rows, cols] (bit b of byte j = col 8j+b)."""
    return np.unpackbits(mask, axis=1, bitorder="little")[:, :cols].astype(bool)


def mma_scale_layout(scales: np.ndarray) -> np.ndarray:
    """Row-wise scales [R, C] (one byte per block) -> the flat byte buffer of
    the block-scaled MMA scale-factor layout, as the cuBLAS documentation
    defines it ("1D block scaling factors layout"): the matrix is padded to
    multiples of 128 rows and 4 columns and cut into 128 x 4 atoms of 512
    bytes, atom (i, j) at byte 512 * (i * ceil(C / 4) + j); inside an atom,
    entry (r, c) is at byte 16 * (r % 32) + 4 * (r // 32) + c. Padding is 0."""
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    R, C = s.shape
    n_rb, n_cb = -(-R // 128), -(-C // 4)
    out = np.zeros(512 * n_rb * n_cb, np.uint8)
    r = np.arange(R, dtype=np.int64)[:, None]
    c = np.arange(C, dtype=np.int64)[None, :]
    i, rr = r // 128, r % 128
    j, cc = c // 4, c % 4
    out[512 * (i * n_cb + j) + 16 * (rr % 32) + 4 * (rr // 32) + cc] = s
    return out


def colwise_operand_k(ends) -> int:
    """K extent of the column-wise operand: every group padded to a multiple
    of 128 rows (four blocks of 32, one scale-atom column)."""
    e = np.asarray(ends, np.int64)
    n = np.diff(np.concatenate([[0], e]))
    return int(np.sum(-(-n // 128)) * 128)


def colwise_operand_layout(codes: np.ndarray, scales: np.ndarray, ends, cols: int, k_alloc: int | None = None):
    """Column-wise E2M1 codes and E8M0 scales (the layout qdq_colwise returns)
    -> the operand of a block-scaled GEMM that contracts over the rows, group
    by group. The pages fix no such layout (parity unpinned); it is this
    library's layout, pinned by hand-computed offsets in the tests:

      K0_g   = sum over j < g of 128 * ceil(n_j / 128)   (group g's first K slot)
      codesT [cols][k_alloc / 2]: the nibble of x[start_g + t, c] is nibble
             (t & 1) of byte c * k_alloc/2 + (K0_g + t) / 2; slots t >= n_g
             up to the group's padded end hold nibble 0
      scales the [cols][k_alloc / 32] E8M0 matrix whose entry (c, K0_g/32 + b)
             is block b of group g in column c (127 for the padding blocks of
             the group), stored in the 128 x 4 atom layout of mma_scale_layout

    Slots past sum of the padded groups (up to k_alloc) are left 0."""
    e = np.asarray(ends, np.int64)
    starts = np.concatenate([[0], e[:-1]])
    n = e - starts
    kpad = -(-n // 128) * 128
    k0 = np.concatenate([[0], np.cumsum(kpad)[:-1]])
    ktot = int(kpad.sum())
    k_alloc = ktot if k_alloc is None else int(k_alloc)
    assert k_alloc >= ktot and k_alloc % 128 == 0
    nib = unpack_nibbles(codes, cols)  # [rows][cols]
    kmat = np.zeros((cols, k_alloc), np.uint8)  # nibble per (column, K slot)
    smat = np.zeros((cols, k_alloc // 32), np.uint8)
    srow = 0
    for g in range(len(e)):
        if n[g] == 0:
            continue
        kmat[:, k0[g]:k0[g] + n[g]] = nib[starts[g]:e[g]].T
        nb = -(-int(n[g]) // 32)
        smat[:, k0[g] // 32:k0[g] // 32 + kpad[g] // 32] = 127
        smat[:, k0[g] // 32:k0[g] // 32 + nb] = scales[srow:srow + nb].T
        srow += nb
    codesT = (kmat[:, 0::2] | (kmat[:, 1::2] << 4)).astype(np.uint8)
    return codesT, mma_scale_layout(smat)


def unpack_nibbles(codes: np.ndarray, cols: int) -> np.ndarray:
    """Packed [rows, ceil(cols/2)] codes -> uint8 [rows, cols] nibbles (low nibble first)."""
    lo = codes & 0x0F
    hi = codes >> 4
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out[:, :cols]


__all__ = [
    "F32", "BF16", "SCALE_PAGE", "SCALE_FLOOR", "lib", "build", "bf16_to_f32", "f32_to_bf16",
    "scale_page", "scale_floor", "qdq_block", "group_ends", "colwise_scale_rows", "qdq_rowwise",
    "qdq_colwise", "ste_bwd", "unpack_bits", "unpack_nibbles", "mma_scale_layout", "qdq8_rowwise",
    "qdq8_colwise", "dual_level_rowwise", "e4m3_value", "e4m3_encode", "colwise_operand_k", "colwise_operand_layout",
]
