"""Torch-facing binding of libmxfp4: the C entry points under the same names.

torch supplies device memory (output allocation) and the current CUDA stream;
every byte of the computation runs in the library's kernels. Inputs must be
CUDA tensors: there is no CPU path.

Tensor conventions follow include/mxfp4.h: x is 2-D [rows, cols] with unit
stride along cols (a 1-D tensor is one row); outputs are contiguous; masks are
bit-packed [rows, ceil(cols/8)] uint8; codes are nibble pairs
[rows, ceil(cols/2)] uint8; row-wise scales [rows, ceil(cols/block)] uint8,
or, with scales_layout="mma", a flat zero-initialised uint8 buffer in the
block-scaled MMA scale-factor layout (128 x 4 atoms; include/mxfp4.h);
column-wise scales [S_bound, cols] uint8 (only the first S rows are written,
S = mxfp4_colwise_scale_rows(...)).
"""
from __future__ import annotations

import dataclasses

import torch

from . import _abi

_DTYPES = {torch.float32: _abi.F32, torch.bfloat16: _abi.BF16}
_MODES = {"page": _abi.SCALE_PAGE, "floor": _abi.SCALE_FLOOR}
_DIRS = {"rowwise": _abi.ROWWISE, "colwise": _abi.COLWISE}
_SCALE_LAYOUTS = {"rowmajor": _abi.SCALES_ROWMAJOR, "mma": _abi.SCALES_MMA}
# element formats: E2M1 (MXFP4) and E4M3 (MXFP8: block 32, scale_mode "floor",
# one code byte per element)
_ELEM_FORMATS = {"e2m1": _abi.ELEM_E2M1, "e4m3": _abi.ELEM_E4M3}
_COL_LAYOUTS = {"rowmajor": _abi.COLS_ROWMAJOR, "mma": _abi.COLS_MMA}


def _elem_format(name: str) -> int:
    if name not in _ELEM_FORMATS:
        raise ValueError(f"elem_format must be one of {tuple(_ELEM_FORMATS)}, got {name!r}")
    return _ELEM_FORMATS[name]


@dataclasses.dataclass
class QDQResult:
    y_row: torch.Tensor | None = None
    y_col: torch.Tensor | None = None
    codes_row: torch.Tensor | None = None
    scales_row: torch.Tensor | None = None
    mask_row: torch.Tensor | None = None
    codes_col: torch.Tensor | None = None
    scales_col: torch.Tensor | None = None
    mask_col: torch.Tensor | None = None
    status: torch.Tensor | None = None
    scales_layout: str = "rowmajor"  # layout of scales_row
    elem_format: str = "e2m1"
    col_layout: str = "rowmajor"  # layout of codes_col / scales_col ("mma": K-major GEMM operand)
    k_alloc: int = 0  # col_layout "mma": K slots per codes_col row


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _as_2d(x: torch.Tensor, name: str = "x") -> torch.Tensor:
    """2-D view of x that the library can address as [rows][ld] with unit
    stride along the columns and ld >= cols. Anything else (a transposed or
    sliced last dimension, rows that overlap such as an expanded tensor with
    row stride 0) is copied first, so that the library never reads outside
    x's storage or with a wrong pitch."""
    if x.ndim == 0:
        raise ValueError(f"{name} must have at least 1 dimension")
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libmxfp4 has no CPU path)")
    if x.dtype not in _DTYPES:
        raise TypeError(f"{name} must be float32 or bfloat16, got {x.dtype}")
    if x.ndim == 1:
        x = x.unsqueeze(0)
    elif x.ndim > 2:
        x = x.reshape(-1, x.shape[-1])
    if not rows_addressable(tuple(x.shape), tuple(x.stride())):
        x = x.contiguous()
    return x


def rows_addressable(shape: tuple, stride: tuple) -> bool:
    """True when a 2-D tensor of this shape and stride is the [rows][ld]
    layout of the C ABI: unit stride along the columns (unless there is only
    one column) and rows that do not overlap (row stride >= cols, unless
    there is only one row)."""
    rows, cols = shape
    return not ((cols > 1 and stride[1] != 1) or (rows > 1 and stride[0] < cols))


def _ld(t: torch.Tensor) -> int:
    """Leading dimension (elements between rows) of a 2-D tensor laid out as
    _as_2d requires; a single row has no pitch and reports its width."""
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _group_args(group_list, group_list_type: int, device):
    if group_list is None:
        return None, 0
    gl = group_list
    if not isinstance(gl, torch.Tensor):
        gl = torch.tensor(list(gl), dtype=torch.int64, device=device)
    if gl.dtype != torch.int64 or not gl.is_cuda or gl.ndim != 1:
        raise ValueError("group_list must be a 1-D int64 CUDA tensor")
    return gl.contiguous(), gl.numel()


def make_args(x: torch.Tensor, *, block: int, scale_factor: float, scale_mode: str, dirs: int,
              group_list=None, group_list_type: int = 0, status: torch.Tensor | None = None,
              elem_format: str = "e2m1") -> _abi.QdqArgs:
    a = _abi.QdqArgs()
    a.x = x.data_ptr()
    a.dtype = _DTYPES[x.dtype]
    a.block = int(block)
    a.rows, a.cols = int(x.shape[0]), int(x.shape[1])
    a.ld = _ld(x)
    a.scale_factor = float(scale_factor)
    if scale_mode not in _MODES:
        raise ValueError(f"scale_mode must be one of {tuple(_MODES)}, got {scale_mode!r}")
    a.scale_mode = _MODES[scale_mode]
    a.dirs = dirs
    if group_list is not None:
        a.group_list = group_list.data_ptr()
        a.num_groups = group_list.numel()
        a.group_list_type = int(group_list_type)
    a.status = _ptr(status)
    a.elem_format = _elem_format(elem_format)
    return a


def colwise_scale_rows_bound(rows: int, num_groups: int, block: int) -> int:
    return _abi.mxfp4_colwise_scale_rows_bound(rows, num_groups, block)


def mxfp4_colwise_scale_rows(group_list, group_list_type: int, rows: int, block: int) -> int:
    """Exact number of column-wise scale rows (copies a device group_list to the host)."""
    if isinstance(group_list, torch.Tensor):
        group_list = group_list.cpu().tolist()
    return _abi.mxfp4_colwise_scale_rows(group_list, group_list_type, rows, block)


def scales_row_bytes(rows: int, cols: int, block: int, scales_layout: str = "rowmajor") -> int:
    if scales_layout not in _SCALE_LAYOUTS:
        raise ValueError(f"scales_layout must be one of {tuple(_SCALE_LAYOUTS)}, got {scales_layout!r}")
    n = _abi.lib().mxfp4_scales_row_bytes(rows, cols, block, _SCALE_LAYOUTS[scales_layout])
    if n < 0:
        raise ValueError("invalid geometry")
    return n


def colwise_operand_k(group_list, group_list_type: int, rows: int) -> int:
    """K extent of the column-wise GEMM operand (col_layout "mma"): exact for
    a host group list (or none), the size-free bound for a device tensor."""
    if isinstance(group_list, torch.Tensor):
        return _abi.lib().mxfp4_colwise_operand_k_bound(rows, group_list.numel())
    k = _abi.mxfp4_colwise_operand_k(None if group_list is None else list(group_list), group_list_type, rows)
    if k < 0:
        raise ValueError("group_list is not a partition of the rows")
    return k


def alloc_outputs(x: torch.Tensor, *, block: int, rowwise: bool, colwise: bool, num_groups: int,
                  emit_values: bool = True, emit_codes: bool = False, emit_mask: bool = False,
                  with_status: bool = False, scales_layout: str = "rowmajor",
                  elem_format: str = "e2m1", col_layout: str = "rowmajor", k_alloc: int | None = None) -> QDQResult:
    rows, cols = x.shape
    dev = x.device
    if col_layout not in _COL_LAYOUTS:
        raise ValueError(f"col_layout must be one of {tuple(_COL_LAYOUTS)}, got {col_layout!r}")
    r = QDQResult(scales_layout=scales_layout, elem_format=elem_format, col_layout=col_layout)
    ccols = cols if _elem_format(elem_format) == _abi.ELEM_E4M3 else (cols + 1) // 2
    u8 = dict(dtype=torch.uint8, device=dev)
    if rowwise:
        if emit_values:
            r.y_row = torch.empty((rows, cols), dtype=x.dtype, device=dev)
        if emit_codes:
            r.codes_row = torch.empty((rows, ccols), **u8)
            if scales_layout == "mma":
                # the padding of the last atoms is never written: zeros
                r.scales_row = torch.zeros((scales_row_bytes(rows, cols, block, "mma"),), **u8)
            else:
                r.scales_row = torch.empty((rows, (cols + block - 1) // block), **u8)
        if emit_mask:
            r.mask_row = torch.empty((rows, (cols + 7) // 8), **u8)
    if colwise:
        if emit_values:
            r.y_col = torch.empty((rows, cols), dtype=x.dtype, device=dev)
        if emit_codes and col_layout == "mma":
            # K slots past the groups and atom rows past cols are not written: zeros
            k = int(k_alloc) if k_alloc is not None else _abi.lib().mxfp4_colwise_operand_k_bound(rows, num_groups)
            r.k_alloc = k
            r.codes_col = torch.zeros((cols, k // 2), **u8)
            r.scales_col = torch.zeros((max(0, _abi.lib().mxfp4_colwise_operand_scale_bytes(cols, k)),), **u8)
        elif emit_codes:
            r.codes_col = torch.empty((rows, ccols), **u8)
            r.scales_col = torch.empty((colwise_scale_rows_bound(rows, num_groups, block), cols), **u8)
        if emit_mask:
            r.mask_col = torch.empty((rows, (cols + 7) // 8), **u8)
    if with_status:
        r.status = torch.empty((1,), dtype=torch.int32, device=dev)
    return r


def _need(t: torch.Tensor, name: str, shape, dtype, device, min_rows: int | None = None) -> None:
    """An output buffer must be a contiguous CUDA tensor of the given shape
    and dtype on x's device (min_rows: at least that many rows instead of
    exactly shape[0])."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    ok = (t.dim() == len(shape) and tuple(t.shape[1:]) == tuple(shape[1:]) and
          (t.shape[0] >= min_rows if min_rows is not None else t.shape[0] == shape[0]))
    if not ok:
        want = f"[>= {min_rows}, {', '.join(map(str, shape[1:]))}]" if min_rows is not None else list(shape)
        raise ValueError(f"{name} has shape {list(t.shape)}, expected {want}")


def _fill_outputs(a: _abi.QdqArgs, r: QDQResult, x: torch.Tensor | None = None) -> None:
    """Copies the output pointers of r into a. With x given, every buffer is
    first checked against the geometry in a (shape, dtype, device, layout), so
    that no kernel can write outside a caller-supplied tensor."""
    if r.scales_layout not in _SCALE_LAYOUTS:
        raise ValueError(f"scales_layout must be one of {tuple(_SCALE_LAYOUTS)}, got {r.scales_layout!r}")
    ys = [t for t in (r.y_row, r.y_col) if t is not None]
    if x is not None:
        rows, cols, blk, dev = a.rows, a.cols, a.block, x.device
        e4m3 = a.elem_format == _abi.ELEM_E4M3
        ccols = cols if e4m3 else (cols + 1) // 2
        nblk = (cols + blk - 1) // blk
        for name in ("y_row", "y_col"):
            t = getattr(r, name)
            if t is None:
                continue
            if not t.is_cuda or t.device != dev or t.dtype != x.dtype or tuple(t.shape) != (rows, cols):
                raise ValueError(f"{name} must be a {x.dtype} CUDA tensor of shape {[rows, cols]} on {dev}")
            if not rows_addressable(tuple(t.shape), tuple(t.stride())):
                raise ValueError(f"{name} must have unit column stride and non-overlapping rows")
        if len(ys) == 2 and _ld(ys[0]) != _ld(ys[1]):
            raise ValueError("y_row and y_col must have the same row stride (one ld_y is passed)")
        u8 = torch.uint8
        if r.col_layout not in _COL_LAYOUTS:
            raise ValueError(f"col_layout must be one of {tuple(_COL_LAYOUTS)}, got {r.col_layout!r}")
        col_mma = r.col_layout == "mma"
        if r.codes_row is not None:
            _need(r.codes_row, "codes_row", (rows, ccols), u8, dev)
        if r.codes_col is not None:
            _need(r.codes_col, "codes_col", (cols, r.k_alloc // 2) if col_mma else (rows, ccols), u8, dev)
        for name in ("mask_row", "mask_col"):
            if getattr(r, name) is not None:
                _need(getattr(r, name), name, (rows, (cols + 7) // 8), u8, dev)
        if r.scales_row is not None:
            if r.scales_layout == "mma":
                t = r.scales_row
                if not t.is_cuda or t.device != dev or t.dtype != u8 or not t.is_contiguous():
                    raise ValueError("scales_row (mma layout) must be a contiguous uint8 CUDA tensor")
                if t.numel() < scales_row_bytes(rows, cols, blk, "mma"):
                    raise ValueError("scales_row (mma layout) is smaller than mxfp4_scales_row_bytes()")
            else:
                _need(r.scales_row, "scales_row", (rows, nblk), u8, dev)
        if r.scales_col is not None and col_mma:
            t = r.scales_col
            if not t.is_cuda or t.device != dev or t.dtype != u8 or not t.is_contiguous():
                raise ValueError("scales_col (mma layout) must be a contiguous uint8 CUDA tensor")
            if t.numel() < _abi.lib().mxfp4_colwise_operand_scale_bytes(cols, r.k_alloc):
                raise ValueError("scales_col (mma layout) is smaller than mxfp4_colwise_operand_scale_bytes()")
        elif r.scales_col is not None:
            _need(r.scales_col, "scales_col", (0, cols), u8, dev,
                  min_rows=colwise_scale_rows_bound(rows, int(a.num_groups) if a.group_list else 0, blk))
        if r.status is not None:
            _need(r.status, "status", (1,), torch.int32, dev)
    a.y_row, a.y_col = _ptr(r.y_row), _ptr(r.y_col)
    a.ld_y = _ld(ys[0]) if ys else a.cols
    a.codes_row, a.scales_row, a.mask_row = _ptr(r.codes_row), _ptr(r.scales_row), _ptr(r.mask_row)
    a.codes_col, a.scales_col, a.mask_col = _ptr(r.codes_col), _ptr(r.scales_col), _ptr(r.mask_col)
    a.scales_row_layout = _SCALE_LAYOUTS[r.scales_layout]
    a.col_layout = _COL_LAYOUTS[r.col_layout]
    a.k_alloc = int(r.k_alloc)


def _check_status(status: torch.Tensor | None, where: str) -> None:
    if status is not None:
        _abi.check(int(status.item()), where + " (group_list)")


def _grad_buffer(out: torch.Tensor | None, g: torch.Tensor, shape, name: str) -> torch.Tensor:
    """The gradient output: a new tensor, or a caller's contiguous tensor of
    grad_out's shape and dtype (the library writes it with grad_out's pitch)."""
    if out is None:
        return torch.empty_like(g)
    if not out.is_cuda or out.device != g.device or out.dtype != g.dtype or not out.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {g.dtype} CUDA tensor on {g.device}")
    if out.numel() != g.numel() or tuple(out.shape) not in (tuple(shape), tuple(g.shape)):
        raise ValueError(f"{name} has shape {list(out.shape)}, expected {list(shape)}")
    return out.view(g.shape)


def mxfp4_qdq_fwd(x: torch.Tensor, *, block: int = 32, scale_factor: float = 6.0, scale_mode: str = "page",
                  rowwise: bool = True, colwise: bool = False, group_list=None, group_list_type: int = 0,
                  emit_values: bool = True, emit_codes: bool = False, emit_mask: bool = False,
                  check: bool | None = None, out: QDQResult | None = None, scales_layout: str = "rowmajor",
                  elem_format: str = "e2m1", col_layout: str = "rowmajor", k_alloc: int | None = None) -> QDQResult:
    """QDQ forward; returns the requested outputs.

    A group_list lives in device memory and is validated by the kernels,
    which write nothing when it is not a partition of the rows. check (the
    default when a group_list is given) synchronises and raises
    MXFP4ArgumentError for such a list. With check=False the call stays
    asynchronous (CUDA-graph capturable) and the outputs are undefined unless
    the returned status tensor reads 0 (MXFP4_OK) once the stream reaches it.
    scales_layout="mma" writes the row-wise scales in the block-scaled MMA
    scale-factor layout. elem_format="e4m3" quantises to MXFP8 (block 32,
    scale_mode "floor"). col_layout="mma" writes the column-wise codes and
    scales as the K-major operand of a GEMM contracting over the rows (each
    group padded to 128 rows; include/mxfp4.h, MXFP4_COLS_MMA); k_alloc
    defaults to the exact K of a host group list, else to the bound."""
    x = _as_2d(x)
    gl, ng = _group_args(group_list, group_list_type, x.device)
    if check is None:
        check = gl is not None and colwise
    dirs = (_abi.ROWWISE if rowwise else 0) | (_abi.COLWISE if colwise else 0)
    if dirs == 0:
        raise ValueError("at least one of rowwise / colwise must be set")
    r = out if out is not None else alloc_outputs(
        x, block=block, rowwise=rowwise, colwise=colwise, num_groups=ng, emit_values=emit_values,
        emit_codes=emit_codes, emit_mask=emit_mask, with_status=check or gl is not None,
        scales_layout=scales_layout, elem_format=elem_format, col_layout=col_layout,
        k_alloc=(k_alloc if k_alloc is not None or col_layout != "mma"
                 else colwise_operand_k(group_list, group_list_type, x.shape[0])))
    if check and r.status is None:
        r.status = torch.empty((1,), dtype=torch.int32, device=x.device)
    a = make_args(x, block=block, scale_factor=scale_factor, scale_mode=scale_mode, dirs=dirs,
                  group_list=gl, group_list_type=group_list_type, status=r.status, elem_format=r.elem_format)
    _fill_outputs(a, r, x)
    _abi.check(_abi.mxfp4_qdq_fwd(a, _stream(x.device)), "mxfp4_qdq_fwd")
    if check:
        _check_status(r.status, "mxfp4_qdq_fwd")
    return r


def mxfp4_ste_bwd(grad_out: torch.Tensor, *, saved_mask: torch.Tensor | None = None,
                  x: torch.Tensor | None = None, clip_grad: bool = True, block: int = 32,
                  scale_factor: float = 6.0, scale_mode: str = "page", direction: str = "rowwise",
                  group_list=None, group_list_type: int = 0, out: torch.Tensor | None = None,
                  elem_format: str = "e2m1", check: bool | None = None,
                  status: torch.Tensor | None = None) -> torch.Tensor:
    """Plain / clipped STE backward. With clip_grad and no saved_mask the mask
    is recomputed from x in the same pass (for elem_format's saturation).

    A group_list only matters when the column-wise mask is recomputed; it is
    then validated by the kernel. check (the default in that case)
    synchronises and raises MXFP4ArgumentError for an invalid list; with
    check=False pass a 1-element int32 CUDA `status` tensor and read it: the
    gradient is undefined unless it holds 0."""
    shape = grad_out.shape
    g = _as_2d(grad_out, "grad_out")
    if not g.is_contiguous():
        g = g.contiguous()
    gi2 = _grad_buffer(out, g, shape, "out")
    if x is not None:
        x2 = _as_2d(x)
        if x2.shape != g.shape or x2.dtype != g.dtype:
            raise ValueError("x and grad_out must have the same shape and dtype")
    else:
        x2 = g  # geometry only; x is not read when the mask is saved
        if clip_grad and saved_mask is None:
            raise ValueError("clip_grad without saved_mask needs x to recompute the mask")
    if saved_mask is not None and clip_grad:
        _need(saved_mask, "saved_mask", (g.shape[0], (g.shape[1] + 7) // 8), torch.uint8, g.device)
    gl, _ = _group_args(group_list, group_list_type, g.device)
    validates = gl is not None and clip_grad and saved_mask is None and direction == "colwise"
    if check is None:
        check = validates
    if validates and status is None:
        if not check:
            raise ValueError("check=False with a group_list needs a status tensor to report the list check")
        status = torch.empty((1,), dtype=torch.int32, device=g.device)
    a = make_args(x2, block=block, scale_factor=scale_factor, scale_mode=scale_mode,
                  dirs=_DIRS[direction], group_list=gl, group_list_type=group_list_type,
                  status=status if validates else None, elem_format=elem_format)
    if x is None:
        a.x = None
    st = _abi.mxfp4_ste_bwd(a, g.data_ptr(), gi2.data_ptr(), g.shape[1], _ptr(saved_mask),
                            int(bool(clip_grad)), _stream(g.device))
    _abi.check(st, "mxfp4_ste_bwd")
    if check and validates:
        _check_status(status, "mxfp4_ste_bwd")
    return gi2.view(shape)


def mxfp4_qdq_fwd_bwd(x: torch.Tensor, grad_out: torch.Tensor, *, grad_direction: str = "rowwise",
                      block: int = 32, scale_factor: float = 6.0, scale_mode: str = "page",
                      rowwise: bool = True, colwise: bool = False, group_list=None, group_list_type: int = 0,
                      emit_values: bool = True, emit_codes: bool = False, emit_mask: bool = False,
                      out: QDQResult | None = None, grad_in: torch.Tensor | None = None,
                      elem_format: str = "e2m1", check: bool | None = None):
    """Fused forward + clipped-STE backward; returns (QDQResult, grad_in).
    A group_list is checked as in mxfp4_qdq_fwd (check defaults to True with
    one; with check=False read the returned status before using anything)."""
    x = _as_2d(x)
    g = _as_2d(grad_out, "grad_out").contiguous()
    if g.shape != x.shape or g.dtype != x.dtype:
        raise ValueError("x and grad_out must have the same shape and dtype")
    gl, ng = _group_args(group_list, group_list_type, x.device)
    if check is None:
        check = gl is not None and colwise
    dirs = (_abi.ROWWISE if rowwise else 0) | (_abi.COLWISE if colwise else 0)
    r = out if out is not None else alloc_outputs(
        x, block=block, rowwise=rowwise, colwise=colwise, num_groups=ng, emit_values=emit_values,
        emit_codes=emit_codes, emit_mask=emit_mask, with_status=check or gl is not None, elem_format=elem_format)
    if check and r.status is None:
        r.status = torch.empty((1,), dtype=torch.int32, device=x.device)
    gi = _grad_buffer(grad_in, g, g.shape, "grad_in")
    a = make_args(x, block=block, scale_factor=scale_factor, scale_mode=scale_mode, dirs=dirs,
                  group_list=gl, group_list_type=group_list_type, status=r.status, elem_format=r.elem_format)
    _fill_outputs(a, r, x)
    st = _abi.mxfp4_qdq_fwd_bwd(a, g.data_ptr(), gi.data_ptr(), g.shape[1], _DIRS[grad_direction],
                                _stream(x.device))
    _abi.check(st, "mxfp4_qdq_fwd_bwd")
    if check:
        _check_status(r.status, "mxfp4_qdq_fwd_bwd")
    return r, gi


def mxfp4_mma_operand(x: torch.Tensor, *, scale_mode: str = "page", scale_factor: float = 6.0,
                      out: QDQResult | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Real MXFP4 operand of a block-scaled GEMM that contracts over x's last
    dimension: (codes [rows, cols/2] as torch.float4_e2m1fn_x2, first element
    in the low nibble; E8M0 scales as torch.float8_e8m0fnu in the 128 x 4 atom
    layout). Block 32 along the contraction; one pass of the row-wise kernel
    writing codes and scales only. Decoding code * 2^(scale - 127) gives the
    fake-quantised values the same call would return as y_row."""
    x2 = _as_2d(x)
    if x2.shape[1] % 2:
        raise ValueError("the contraction dimension must be even (two E2M1 codes per byte)")
    r = mxfp4_qdq_fwd(x2, block=32, scale_factor=scale_factor, scale_mode=scale_mode, rowwise=True,
                      emit_values=False, emit_codes=True, out=out, scales_layout="mma")
    return r.codes_row.view(torch.float4_e2m1fn_x2), r.scales_row.view(torch.float8_e8m0fnu)


def mxfp4_colwise_mma_operand(x: torch.Tensor, *, group_list=None, group_list_type: int = 0,
                              scale_mode: str = "page", scale_factor: float = 6.0, k_alloc: int | None = None,
                              check: bool | None = None):
    """Real MXFP4 operand of a block-scaled GEMM that contracts over x's rows,
    per group (the weight-gradient direction): returns (codes [cols,
    k_alloc/2] as torch.float4_e2m1fn_x2, K-major, first row in the low
    nibble; E8M0 scales as torch.float8_e8m0fnu in the 128 x 4 atom layout of
    the [cols][k_alloc/32] scale matrix; k_alloc). Group g occupies K slots
    [K0_g, K0_g + 128 ceil(n_g/128)) with K0_g the sum of the earlier groups'
    padded sizes; the padding codes are 0. A group_list given as a host
    sequence fixes k_alloc exactly; a device tensor uses the bound."""
    x2 = _as_2d(x)
    r = mxfp4_qdq_fwd(x2, block=32, scale_factor=scale_factor, scale_mode=scale_mode, rowwise=False,
                      colwise=True, group_list=group_list, group_list_type=group_list_type, emit_values=False,
                      emit_codes=True, col_layout="mma", k_alloc=k_alloc, check=check)
    return r.codes_col.view(torch.float4_e2m1fn_x2), r.scales_col.view(torch.float8_e8m0fnu), r.k_alloc


_GMM_MODES = {"m": _abi.GMM_GROUP_M, "k": _abi.GMM_GROUP_K}


def mxfp4_grouped_gemm(a: torch.Tensor, a_scales: torch.Tensor, b: torch.Tensor, b_scales: torch.Tensor,
                       group_list, *, k: int, group_mode: str = "m", elem_format: str = "e2m1",
                       group_list_type: int = 0, k_rows: int | None = None, out_dtype=torch.float32,
                       check: bool | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """Grouped block-scaled GEMM D = A B^T on the tensor cores (include/mxfp4.h,
    mxfp4_grouped_gemm), on operands as this library emits them.

    a: [m, k/2] (E2M1) or [m, k] (E4M3) uint8 codes, K-major; a_scales: the
    MMA-layout E8M0 scales of A. group_mode "m": the group list splits the
    m rows; b is [G, n, row bytes] or [G * n, row bytes], b_scales G
    consecutive MMA-layout scale buffers; D is [m, n]. group_mode "k": A and
    B are column-wise operands (col_layout "mma", k = their k_alloc), the
    group list splits k_rows rows; D is [G, m, n]. check (the default)
    synchronises and raises for an invalid group list."""
    fmt = _elem_format(elem_format)
    if group_mode not in _GMM_MODES:
        raise ValueError(f"group_mode must be 'm' or 'k', got {group_mode!r}")
    for t, name in ((a, "a"), (a_scales, "a_scales"), (b, "b"), (b_scales, "b_scales")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype not in (torch.uint8, torch.float4_e2m1fn_x2,
                                                                                 torch.float8_e4m3fn, torch.float8_e8m0fnu):
            raise ValueError(f"{name} must be a CUDA uint8 (or fp4 / fp8 / e8m0) tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    a8, b8 = a.view(torch.uint8), b.view(torch.uint8)
    kb = k // 2 if fmt == _abi.ELEM_E2M1 else k
    if k <= 0 or k % 128:
        raise ValueError("k must be a positive multiple of 128")
    a8 = a8.reshape(-1, a8.shape[-1])
    b8 = b8.reshape(-1, b8.shape[-1])
    if a8.shape[1] < kb or b8.shape[1] < kb:
        raise ValueError("operand rows are shorter than k")
    gl, ng = _group_args(group_list, group_list_type, a.device)
    if gl is None:
        raise ValueError("a group_list is required (one group: [rows])")
    m = a8.shape[0]
    gk = group_mode == "k"
    if gk:
        n = b8.shape[0]
        if k_rows is None:
            raise ValueError("group_mode 'k' needs k_rows (the rows the group list partitions)")
        shape = (ng, m, n)
    else:
        if b8.shape[0] % ng:
            raise ValueError("b must stack num_groups matrices of n rows")
        n = b8.shape[0] // ng
        shape = (m, n)
    if check is None:
        check = True
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    d = out if out is not None else torch.empty(shape, dtype=out_dtype, device=a.device)
    if tuple(d.shape) != shape or d.dtype != out_dtype or not d.is_contiguous():
        raise ValueError(f"out must be a contiguous {out_dtype} tensor of shape {list(shape)}")
    st = torch.empty((1,), dtype=torch.int32, device=a.device)
    g = _abi.GmmArgs()
    g.elem_format = fmt
    g.group_mode = _GMM_MODES[group_mode]
    g.m, g.n, g.k = m, n, int(k)
    g.a, g.lda, g.a_scales = a8.data_ptr(), a8.stride(0), a_scales.data_ptr()
    g.b, g.ldb, g.b_scales = b8.data_ptr(), b8.stride(0), b_scales.data_ptr()
    g.group_list, g.num_groups, g.group_list_type = gl.data_ptr(), ng, int(group_list_type)
    g.d_dtype = _DTYPES[out_dtype]
    g.k_rows = int(k_rows) if gk else 0
    g.d, g.ldd = d.data_ptr(), n
    g.status = st.data_ptr()
    _abi.check(_abi.mxfp4_grouped_gemm(g, _stream(a.device)), "mxfp4_grouped_gemm")
    if check:
        _check_status(st, "mxfp4_grouped_gemm")
    return d


@dataclasses.dataclass
class DualLevelResult:
    y: torch.Tensor | None = None
    codes: torch.Tensor | None = None
    scales0: torch.Tensor | None = None
    scales1: torch.Tensor | None = None
    mask: torch.Tensor | None = None


def mxfp4_dual_level_qdq(x: torch.Tensor, *, level0_block: int = 512, scale_factor: float = 6.0,
                         scale_mode: str = "page", emit_values: bool = True, emit_codes: bool = True,
                         emit_mask: bool = False, out: DualLevelResult | None = None) -> DualLevelResult:
    """Dual-level MX quantisation of a bf16 tensor along its last dimension
    (include/mxfp4.h, mxfp4_dual_level_qdq): fp32 level-0 scales
    [rows, ceil(cols/level0_block)], E8M0 level-1 scales [rows, ceil(cols/32)],
    packed E2M1 codes, and on request the dequantised bf16 values and the
    bit-packed saturation mask (which mxfp4_ste_bwd takes as saved_mask).
    Asynchronous on the current stream."""
    x = _as_2d(x)
    if x.dtype != torch.bfloat16:
        raise TypeError("dual-level quantisation takes bfloat16 input")
    if scale_mode not in _MODES:
        raise ValueError(f"scale_mode must be 'page' or 'floor', got {scale_mode!r}")
    rows, cols = x.shape
    dev = x.device
    r = out if out is not None else DualLevelResult(
        y=torch.empty((rows, cols), dtype=torch.bfloat16, device=dev) if emit_values else None,
        codes=torch.empty((rows, (cols + 1) // 2), dtype=torch.uint8, device=dev) if emit_codes else None,
        scales0=torch.empty((rows, -(-cols // max(level0_block, 1))), dtype=torch.float32, device=dev),
        scales1=torch.empty((rows, -(-cols // 32)), dtype=torch.uint8, device=dev),
        mask=torch.empty((rows, (cols + 7) // 8), dtype=torch.uint8, device=dev) if emit_mask else None)
    if r.y is not None:
        _need(r.y, "y", (rows, cols), torch.bfloat16, dev)
    for t, name, shape, dt in ((r.codes, "codes", (rows, (cols + 1) // 2), torch.uint8),
                               (r.scales0, "scales0", (rows, -(-cols // max(level0_block, 1))), torch.float32),
                               (r.scales1, "scales1", (rows, -(-cols // 32)), torch.uint8),
                               (r.mask, "mask", (rows, (cols + 7) // 8), torch.uint8)):
        if t is not None:
            _need(t, name, shape, dt, dev)
    a = _abi.DualLevelArgs()
    a.x, a.dtype, a.level0_block = x.data_ptr(), _abi.BF16, int(level0_block)
    a.rows, a.cols, a.ld = rows, cols, _ld(x)
    a.scale_factor, a.scale_mode = float(scale_factor), _MODES[scale_mode]
    a.y, a.ld_y = _ptr(r.y), cols
    a.codes, a.scales0, a.scales1, a.mask = _ptr(r.codes), _ptr(r.scales0), _ptr(r.scales1), _ptr(r.mask)
    _abi.check(_abi.mxfp4_dual_level_qdq(a, _stream(dev)), "mxfp4_dual_level_qdq")
    return r
