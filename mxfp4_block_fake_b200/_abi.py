"""ctypes view of libmxfp4.so (the C ABI declared in include/mxfp4.h).

Argument marshalling only: the structure below mirrors `mxfp4_qdq_args`
field for field, and every entry point is bound with its exact C signature.
The library must have been built (python -m mxfp4_block_fake_b200.build);
there is no fallback of any kind when it is missing.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmxfp4.so")

OK, EINVAL, EUNSUPPORTED, ECUDA = 0, 1, 2, 3
F32, BF16 = 0, 1
SCALE_PAGE, SCALE_FLOOR = 0, 1
ROWWISE, COLWISE = 1, 2
SCALES_ROWMAJOR, SCALES_MMA = 0, 1
COLS_ROWMAJOR, COLS_MMA = 0, 1
ELEM_E2M1, ELEM_E4M3 = 0, 1
MAX_GROUPS = 4096
ABI_VERSION = 5

# Every symbol include/mxfp4.h declares.
EXPORTS = (
    "mxfp4_qdq_fwd",
    "mxfp4_ste_bwd",
    "mxfp4_qdq_fwd_bwd",
    "mxfp4_colwise_scale_rows",
    "mxfp4_colwise_scale_rows_bound",
    "mxfp4_scales_row_bytes",
    "mxfp4_colwise_operand_k",
    "mxfp4_colwise_operand_k_bound",
    "mxfp4_colwise_operand_scale_bytes",
    "mxfp4_grouped_gemm",
    "mxfp4_dual_level_qdq",
    "mxfp4_status_string",
    "mxfp4_abi_version",
)


class QdqArgs(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("ld", ctypes.c_int64),
        ("scale_factor", ctypes.c_float),
        ("scale_mode", ctypes.c_int32),
        ("dirs", ctypes.c_uint32),
        ("group_list_type", ctypes.c_int32),
        ("group_list", ctypes.c_void_p),
        ("num_groups", ctypes.c_int64),
        ("status", ctypes.c_void_p),
        ("y_row", ctypes.c_void_p),
        ("y_col", ctypes.c_void_p),
        ("ld_y", ctypes.c_int64),
        ("codes_row", ctypes.c_void_p),
        ("scales_row", ctypes.c_void_p),
        ("mask_row", ctypes.c_void_p),
        ("codes_col", ctypes.c_void_p),
        ("scales_col", ctypes.c_void_p),
        ("mask_col", ctypes.c_void_p),
        ("scales_row_layout", ctypes.c_int32),
        ("elem_format", ctypes.c_int32),
        ("col_layout", ctypes.c_int32),
        ("k_alloc", ctypes.c_int64),
    ]


GMM_GROUP_M, GMM_GROUP_K = 0, 1


class GmmArgs(ctypes.Structure):
    _fields_ = [
        ("elem_format", ctypes.c_int32),
        ("group_mode", ctypes.c_int32),
        ("m", ctypes.c_int64),
        ("n", ctypes.c_int64),
        ("k", ctypes.c_int64),
        ("a", ctypes.c_void_p),
        ("lda", ctypes.c_int64),
        ("a_scales", ctypes.c_void_p),
        ("b", ctypes.c_void_p),
        ("ldb", ctypes.c_int64),
        ("b_scales", ctypes.c_void_p),
        ("group_list", ctypes.c_void_p),
        ("num_groups", ctypes.c_int64),
        ("group_list_type", ctypes.c_int32),
        ("d_dtype", ctypes.c_int32),
        ("k_rows", ctypes.c_int64),
        ("d", ctypes.c_void_p),
        ("ldd", ctypes.c_int64),
        ("status", ctypes.c_void_p),
    ]


class DualLevelArgs(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("level0_block", ctypes.c_int32),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("ld", ctypes.c_int64),
        ("scale_factor", ctypes.c_float),
        ("scale_mode", ctypes.c_int32),
        ("y", ctypes.c_void_p),
        ("ld_y", ctypes.c_int64),
        ("codes", ctypes.c_void_p),
        ("scales0", ctypes.c_void_p),
        ("scales1", ctypes.c_void_p),
        ("mask", ctypes.c_void_p),
    ]


class MXFP4Error(RuntimeError):
    """A libmxfp4 call returned a non-OK status."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class MXFP4ArgumentError(MXFP4Error, ValueError):
    """MXFP4_EINVAL / MXFP4_EUNSUPPORTED: the arguments were rejected."""


_lib: ctypes.CDLL | None = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libmxfp4.so not found at {LIB_PATH}; build it with "
            "`python -m mxfp4_block_fake_b200.build` (nvcc, sm_100a)"
        )
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32
    A = ctypes.POINTER(QdqArgs)
    L.mxfp4_qdq_fwd.argtypes = [A, P]
    L.mxfp4_qdq_fwd.restype = i32
    L.mxfp4_ste_bwd.argtypes = [A, P, P, i64, P, i32, P]
    L.mxfp4_ste_bwd.restype = i32
    L.mxfp4_qdq_fwd_bwd.argtypes = [A, P, P, i64, u32, P]
    L.mxfp4_qdq_fwd_bwd.restype = i32
    L.mxfp4_colwise_scale_rows.argtypes = [P, i64, i32, i64, i32]
    L.mxfp4_colwise_scale_rows.restype = i64
    L.mxfp4_colwise_scale_rows_bound.argtypes = [i64, i64, i32]
    L.mxfp4_colwise_scale_rows_bound.restype = i64
    L.mxfp4_scales_row_bytes.argtypes = [i64, i64, i32, i32]
    L.mxfp4_scales_row_bytes.restype = i64
    L.mxfp4_colwise_operand_k.argtypes = [P, i64, i32, i64]
    L.mxfp4_colwise_operand_k.restype = i64
    L.mxfp4_colwise_operand_k_bound.argtypes = [i64, i64]
    L.mxfp4_colwise_operand_k_bound.restype = i64
    L.mxfp4_colwise_operand_scale_bytes.argtypes = [i64, i64]
    L.mxfp4_colwise_operand_scale_bytes.restype = i64
    L.mxfp4_grouped_gemm.argtypes = [ctypes.POINTER(GmmArgs), P]
    L.mxfp4_grouped_gemm.restype = i32
    L.mxfp4_dual_level_qdq.argtypes = [ctypes.POINTER(DualLevelArgs), P]
    L.mxfp4_dual_level_qdq.restype = i32
    L.mxfp4_status_string.argtypes = [i32]
    L.mxfp4_status_string.restype = ctypes.c_char_p
    L.mxfp4_abi_version.argtypes = []
    L.mxfp4_abi_version.restype = i32
    if L.mxfp4_abi_version() != ABI_VERSION:
        raise ImportError(f"libmxfp4.so ABI {L.mxfp4_abi_version()} != binding ABI {ABI_VERSION}")
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().mxfp4_status_string(status).decode()


def check(status: int, where: str) -> None:
    if status == OK:
        return
    if status in (EINVAL, EUNSUPPORTED):
        raise MXFP4ArgumentError(status, where)
    raise MXFP4Error(status, where)


# Thin same-name wrappers of the C entry points (pointers are plain ints).

def mxfp4_qdq_fwd(args: QdqArgs, stream: int) -> int:
    return lib().mxfp4_qdq_fwd(ctypes.byref(args), stream)


def mxfp4_ste_bwd(geom: QdqArgs, grad_out: int, grad_in: int, ld_grad: int, saved_mask: int | None,
                  clip_grad: int, stream: int) -> int:
    return lib().mxfp4_ste_bwd(ctypes.byref(geom), grad_out, grad_in, ld_grad, saved_mask, clip_grad, stream)


def mxfp4_qdq_fwd_bwd(args: QdqArgs, grad_out: int, grad_in: int, ld_grad: int, grad_dir: int,
                      stream: int) -> int:
    return lib().mxfp4_qdq_fwd_bwd(ctypes.byref(args), grad_out, grad_in, ld_grad, grad_dir, stream)


def mxfp4_colwise_scale_rows(host_group_list, group_list_type: int, rows: int, block: int) -> int:
    """host_group_list: a sequence of ints (host memory)."""
    if host_group_list is None:
        return lib().mxfp4_colwise_scale_rows(None, 0, group_list_type, rows, block)
    n = len(host_group_list)
    arr = (ctypes.c_int64 * n)(*[int(v) for v in host_group_list])
    return lib().mxfp4_colwise_scale_rows(arr, n, group_list_type, rows, block)


def mxfp4_colwise_scale_rows_bound(rows: int, num_groups: int, block: int) -> int:
    return lib().mxfp4_colwise_scale_rows_bound(rows, num_groups, block)


def mxfp4_colwise_operand_k(host_group_list, group_list_type: int, rows: int) -> int:
    """host_group_list: a sequence of ints (host memory), or None for one group."""
    if host_group_list is None:
        return lib().mxfp4_colwise_operand_k(None, 0, group_list_type, rows)
    n = len(host_group_list)
    arr = (ctypes.c_int64 * n)(*[int(v) for v in host_group_list])
    return lib().mxfp4_colwise_operand_k(arr, n, group_list_type, rows)


def mxfp4_grouped_gemm(args: GmmArgs, stream: int) -> int:
    return lib().mxfp4_grouped_gemm(ctypes.byref(args), stream)


def mxfp4_dual_level_qdq(args: DualLevelArgs, stream: int) -> int:
    return lib().mxfp4_dual_level_qdq(ctypes.byref(args), stream)
