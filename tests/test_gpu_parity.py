"""GPU parity: the CUDA path (called through the C ABI) against the CPU oracle.

Tolerance: 0 ULP. Every dequantised value is exactly representable, so the bf16
/ fp32 outputs, the packed E2M1 codes, the E8M0 scales, the saturation
bitmasks and the STE gradients must match the oracle byte for byte.

Shapes span several tiles plus ragged tails (rows not a multiple of the block,
cols not a multiple of the block, of 8, or of the tile width), strided and
unaligned inputs (the generic kernels), empty tensors, group lists with empty
groups and partial tail blocks, every finite bf16 value as element and as
block maximum. The workloads at their full sizes, compared in full, are in
test_gpu_full_size.py.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import MXFP4ArgumentError, ops, workloads as W

pytestmark = pytest.mark.gpu

MODES = {"page": O.SCALE_PAGE, "floor": O.SCALE_FLOOR}


def np_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy().view(np.uint32)
    return t.numpy()


def oracle_in(x: torch.Tensor) -> np.ndarray:
    x = x.contiguous()
    return np_bits(x) if x.dtype == torch.bfloat16 else x.numpy()


def ora_bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def check_dir(res: ops.QDQResult, ora: dict, d: str, cols: int, srows: int | None = None, label=""):
    y, codes, scales, mask = (getattr(res, f"{k}_{d}") for k in ("y", "codes", "scales", "mask"))
    if y is not None:
        g = np_bits(y)
        e = ora_bits(ora["y"])
        bad = np.argwhere(g != e)
        assert bad.size == 0, f"{label} y_{d}: {len(bad)} mismatches, first {bad[:3].tolist()} " \
                              f"gpu {g[tuple(bad[0])]:#x} oracle {e[tuple(bad[0])]:#x}"
    if codes is not None:
        assert np.array_equal(np_bits(codes), ora["codes"]), f"{label} codes_{d}"
    if scales is not None:
        s = ora["scales"].shape[0] if srows is None else srows
        assert np.array_equal(np_bits(scales)[:s], ora["scales"][:s]), f"{label} scales_{d}"
    if mask is not None:
        assert np.array_equal(np_bits(mask), ora["mask"]), f"{label} mask_{d}"


def run_both(x: torch.Tensor, *, block: int, mode: str, rowwise: bool, colwise: bool, counts=None,
             gl_type: int = 0, sf: float = 6.0, xdev: torch.Tensor | None = None):
    xd = x.cuda() if xdev is None else xdev
    gl = None
    ends = None
    if counts is not None:
        counts = np.asarray(counts, np.int64)
        ends = np.cumsum(counts)
        gl = torch.tensor(counts if gl_type == 1 else ends, dtype=torch.int64, device="cuda")
    res = ops.mxfp4_qdq_fwd(xd, block=block, scale_factor=sf, scale_mode=mode, rowwise=rowwise, colwise=colwise,
                            group_list=gl, group_list_type=gl_type, emit_codes=True, emit_mask=True, check=True)
    torch.cuda.synchronize()
    xo = oracle_in(x)
    out = {}
    if rowwise:
        out["row"] = O.qdq_rowwise(xo, block, sf, MODES[mode])
    if colwise:
        out["col"] = O.qdq_colwise(xo, block, sf, MODES[mode], ends=ends)
    return res, out


SHAPES = [(300, 1024), (37, 1000), (129, 136), (1, 64), (64, 4096), (5, 999), (33, 77), (2, 8)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("shape", SHAPES)
def test_rowwise(dtype, block, mode, shape):
    x = W.mixed(*shape, dtype=dtype, seed=hash(shape) % 1000)
    res, ora = run_both(x, block=block, mode=mode, rowwise=True, colwise=False)
    check_dir(res, ora["row"], "row", shape[1], label=f"{shape}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("shape", SHAPES)
def test_colwise_and_dual(dtype, block, mode, shape):
    x = W.mixed(*shape, dtype=dtype, seed=1 + hash(shape) % 1000)
    res, ora = run_both(x, block=block, mode=mode, rowwise=False, colwise=True)
    check_dir(res, ora["col"], "col", shape[1], label=f"col {shape}")
    res, ora = run_both(x, block=block, mode=mode, rowwise=True, colwise=True)
    check_dir(res, ora["row"], "row", shape[1], label=f"dual {shape}")
    check_dir(res, ora["col"], "col", shape[1], label=f"dual {shape}")


GROUPS = [
    [0, 45, 32, 0, 1, 70, 0],          # empty groups, partial tails, a 1-row group
    [300],                               # one group
    [0, 0, 300],
    [31, 33, 64, 128, 44],
    [1] * 40 + [260],
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("gl_type", [0, 1])
@pytest.mark.parametrize("gi", range(len(GROUPS)))
@pytest.mark.parametrize("cols", [256, 200, 99])
def test_grouped_colwise_and_dual(dtype, block, gl_type, gi, cols):
    counts = GROUPS[gi]
    rows = sum(counts)
    x = W.mixed(rows, cols, dtype=dtype, seed=100 + gi)
    mode = "page" if gi % 2 == 0 else "floor"
    res, ora = run_both(x, block=block, mode=mode, rowwise=True, colwise=True, counts=counts, gl_type=gl_type)
    check_dir(res, ora["row"], "row", cols, label="grouped")
    check_dir(res, ora["col"], "col", cols, label="grouped")
    assert int(res.status.item()) == 0


def test_moe_group_recipe_reduced():
    counts = W.moe_group_counts(4096, 256, seed=4).numpy()
    x = W.moe_grouped(4096, 512, 256, seed=4)[0]
    res, ora = run_both(x, block=32, mode="page", rowwise=True, colwise=True, counts=counts)
    check_dir(res, ora["row"], "row", 512)
    check_dir(res, ora["col"], "col", 512)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dirs", [(True, False), (False, True), (True, True)])
def test_strided_and_unaligned_inputs(dtype, dirs):
    big = W.mixed(70, 272, dtype=dtype, seed=5).cuda()
    for view in (big[:, 8:264], big[:, 3:259], big[1:, 1:200]):
        x = view.cpu()
        res, ora = run_both(x, block=32, mode="page", rowwise=dirs[0], colwise=dirs[1], xdev=view)
        if dirs[0]:
            check_dir(res, ora["row"], "row", x.shape[1], label="strided")
        if dirs[1]:
            check_dir(res, ora["col"], "col", x.shape[1], label="strided")


@pytest.mark.parametrize("offsets", [(0, 0), (4, 1), (4, 0), (0, 3)])
@pytest.mark.parametrize("rows,cols,counts", [(96, 512, None), (70, 768, [20, 0, 37, 13]), (64, 256, [64])])
def test_padded_and_offset_outputs(offsets, rows, cols, counts):
    """Outputs in padded rows (ld_y > cols) and code/mask buffers starting at
    byte offsets: tensor-map stores where they can address the output,
    thread copies where they cannot; both must give the oracle's bytes."""
    co, mo = offsets
    x = W.mixed(rows, cols, dtype=torch.bfloat16, seed=31)
    xd = x.cuda()
    dev = xd.device
    u8 = dict(dtype=torch.uint8, device=dev)

    def flat(n, off):
        return torch.full((n + off,), 0xA5, **u8)[off:]

    ng = 0 if counts is None else len(counts)
    r = ops.QDQResult()
    r.y_row = torch.empty((rows, cols + 8), dtype=torch.bfloat16, device=dev)[:, :cols]
    r.y_col = torch.empty((rows, cols + 8), dtype=torch.bfloat16, device=dev)[:, :cols]
    r.codes_row = flat(rows * cols // 2, co).view(rows, cols // 2)
    r.codes_col = flat(rows * cols // 2, co).view(rows, cols // 2)
    r.mask_row = flat(rows * cols // 8, mo).view(rows, cols // 8)
    r.mask_col = flat(rows * cols // 8, mo).view(rows, cols // 8)
    r.scales_row = torch.empty((rows, cols // 32), **u8)
    r.scales_col = torch.empty((ops.colwise_scale_rows_bound(rows, ng, 32), cols), **u8)
    r.status = torch.empty((1,), dtype=torch.int32, device=dev)
    gl = None if counts is None else torch.tensor(counts, dtype=torch.int64, device=dev)
    ops.mxfp4_qdq_fwd(xd, rowwise=True, colwise=True, group_list=gl, group_list_type=1, emit_codes=True,
                      emit_mask=True, out=r, check=True)
    torch.cuda.synchronize()
    xo = oracle_in(x)
    ends = None if counts is None else np.cumsum(np.asarray(counts, np.int64))
    check_dir(r, O.qdq_rowwise(xo, 32, 6.0, O.SCALE_PAGE), "row", cols, label="padded/offset")
    check_dir(r, O.qdq_colwise(xo, 32, 6.0, O.SCALE_PAGE, ends=ends), "col", cols, label="padded/offset")


MMA_CASES = [
    # (dtype, block, rows, cols, colwise, counts, scales byte offset)
    (torch.bfloat16, 32, 300, 1024, False, None, 0),       # staged, row-wise only
    (torch.bfloat16, 32, 300, 1024, True, None, 0),        # staged, dual
    (torch.bfloat16, 32, 261, 1000, True, [100, 0, 61, 100], 0),  # staged, grouped, ragged
    (torch.bfloat16, 32, 300, 200, True, None, 0),         # staged, 7 blocks per row
    (torch.bfloat16, 32, 300, 1024, True, None, 1),        # staged, unaligned scales buffer
    (torch.bfloat16, 128, 300, 1024, True, None, 0),       # staged block 128
    (torch.bfloat16, 128, 130, 640, False, None, 0),       # block 128 row-wise
    (torch.float32, 32, 129, 136, True, None, 0),          # register-tile kernel
    (torch.float32, 128, 260, 512, False, None, 0),        # register-tile kernel, block 128
    (torch.bfloat16, 32, 5, 999, True, None, 0),           # scalar kernels (odd cols)
]


@pytest.mark.parametrize("case", MMA_CASES)
def test_mma_scale_layout(case):
    """Row-wise scales written straight into the block-scaled MMA layout
    (128 x 4 atoms) equal the oracle's row-major scales placed by the
    oracle's layout; padding bytes stay untouched; the other outputs are the
    same as with the row-major layout."""
    dtype, block, rows, cols, colwise, counts, soff = case
    x = W.mixed(rows, cols, dtype=dtype, seed=41 + rows)
    xd = x.cuda()
    ng = 0 if counts is None else len(counts)
    r = ops.alloc_outputs(xd, block=block, rowwise=True, colwise=colwise, num_groups=ng, emit_codes=True,
                          emit_mask=True, with_status=True, scales_layout="mma")
    n = r.scales_row.numel()
    r.scales_row = torch.zeros((n + soff,), dtype=torch.uint8, device=xd.device)[soff:]
    gl = None if counts is None else torch.tensor(counts, dtype=torch.int64, device=xd.device)
    ops.mxfp4_qdq_fwd(xd, block=block, rowwise=True, colwise=colwise, group_list=gl, group_list_type=1,
                      emit_codes=True, emit_mask=True, out=r, check=True)
    torch.cuda.synchronize()
    xo = oracle_in(x)
    ora = O.qdq_rowwise(xo, block, 6.0, O.SCALE_PAGE)
    got = r.scales_row.cpu().numpy()
    exp = O.mma_scale_layout(ora["scales"])
    assert got.size == exp.size
    bad = np.flatnonzero(got != exp)
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:4].tolist()}"
    r.scales_row = None
    check_dir(r, ora, "row", cols, label="mma layout")
    if colwise:
        ends = None if counts is None else np.cumsum(np.asarray(counts, np.int64))
        check_dir(r, O.qdq_colwise(xo, block, 6.0, O.SCALE_PAGE, ends=ends), "col", cols, label="mma layout")


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("mnk", [(256, 384, 2048), (192, 256, 1024)])
def test_mma_operands_in_a_real_fp4_gemm(mode, mnk):
    """The packed codes and MMA-layout scales, fed to a block-scaled FP4
    tensor-core GEMM (torch's scaled_mm, MXFP4: E2M1 data, E8M0 scales per 32
    along K, 128 x 4 scale atoms), give the product of the fake-quantised
    matrices: real quantisation equals fake quantisation. Reference: the
    oracle's dequantised values multiplied in float64. Bound: the bf16 output
    rounding (2^-8 relative) plus fp32 accumulation over K terms
    (K 2^-23 of the sum of |products|)."""
    from torch.nn.functional import ScalingType, SwizzleType, scaled_mm
    M, N, K = mnk
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16)
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(N + 1)).to(torch.bfloat16)
    cx, sx = ops.mxfp4_mma_operand(x.cuda(), scale_mode=mode)
    cw, sw = ops.mxfp4_mma_operand(w.cuda(), scale_mode=mode)
    out = scaled_mm(cx, cw.t(), sx, ScalingType.BlockWise1x32, sw, ScalingType.BlockWise1x32,
                    swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                    output_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    yx = O.bf16_to_f32(O.qdq_rowwise(oracle_in(x), 32, 6.0, MODES[mode])["y"]).astype(np.float64)
    yw = O.bf16_to_f32(O.qdq_rowwise(oracle_in(w), 32, 6.0, MODES[mode])["y"]).astype(np.float64)
    ref = yx @ yw.T
    mag = np.abs(yx) @ np.abs(yw).T
    err = np.abs(out.float().cpu().numpy().astype(np.float64) - ref)
    bound = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * mag
    assert np.all(err <= bound), f"max err/bound {float((err / bound).max()):.3f}"


@pytest.mark.parametrize("sf", [1.0, 4.0, 7.5, 0.75, 3.0e-38, 1.0e30])
def test_scale_factors_page_mode(sf):
    x = W.mixed(64, 512, seed=6)
    res, ora = run_both(x, block=32, mode="page", rowwise=True, colwise=True, sf=sf)
    check_dir(res, ora["row"], "row", 512)
    check_dir(res, ora["col"], "col", 512)


def bf16_sweep_block32() -> np.ndarray:
    """Rows of 32-element blocks: every bf16 value as block maximum (with a
    neighbour and its negation), and as element under fixed maxima."""
    allv = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rows = []
    for shift in (0, 1, 3):
        blk = np.zeros((65536, 32), np.uint16)
        blk[:, 0] = allv
        blk[:, 1] = np.where((allv & 0x7F80) >= (shift << 7), allv - (shift << 7), allv)
        blk[:, 2] = allv ^ 0x8000
        blk[:, 5] = 0x3F80
        rows.append(blk)
    for mx in (0x40C0, 0x4090, 0x3F80, 0x40F8, 0x0010, 0x7F7F):
        blk = np.zeros((65536, 32), np.uint16)
        blk[:, 0] = mx
        blk[:, 7] = allv
        rows.append(blk)
    return np.concatenate(rows)


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_every_bf16_value_as_element_and_as_block_max(mode):
    xb = bf16_sweep_block32()
    x = torch.from_numpy(xb.view(np.int16).copy()).view(torch.bfloat16)
    res, ora = run_both(x, block=32, mode=mode, rowwise=True, colwise=False)
    check_dir(res, ora["row"], "row", 32, label="bf16 sweep")


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("scales", [False, True])
def test_every_bf16_value_values_only(mode, scales):
    """The sweep with dequantised values alone (and with scales): the row-wise
    kernel for that output mix differs from the one with codes and masks."""
    xb = bf16_sweep_block32().reshape(-1, 256)
    x = torch.from_numpy(xb.view(np.int16).copy()).view(torch.bfloat16)
    xd = x.cuda()
    r = ops.QDQResult()
    r.y_row = torch.empty_like(xd)
    if scales:
        r.scales_row = torch.empty((xd.shape[0], 8), dtype=torch.uint8, device=xd.device)
    ops.mxfp4_qdq_fwd(xd, block=32, scale_mode=mode, rowwise=True, out=r)
    torch.cuda.synchronize()
    ora = O.qdq_rowwise(oracle_in(x), 32, 6.0, MODES[mode])
    check_dir(r, ora, "row", 256, label="values only")


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("counts", [None, [32], [16, 0, 16]])
def test_every_bf16_value_block32_along_columns(mode, counts):
    """The block-32 sweep laid along columns (the transpose: 32 rows, one
    column per sweep block) through the staged dual kernel, every output of
    both directions: every finite bf16 value as element and as column-block
    maximum, in the low and the high half of a 32-bit word. Ungrouped, with
    one group, and with groups that cut every column block into two tails
    (the group-tail path of the kernel)."""
    xb = np.ascontiguousarray(bf16_sweep_block32().T)  # [32, 589824]
    x = torch.from_numpy(xb.view(np.int16).copy()).view(torch.bfloat16)
    res, ora = run_both(x, block=32, mode=mode, rowwise=True, colwise=True, counts=counts)
    check_dir(res, ora["row"], "row", xb.shape[1], label="bf16 sweep along columns")
    check_dir(res, ora["col"], "col", xb.shape[1], label="bf16 sweep along columns")


def codes_only(x: torch.Tensor, mode: str, layout: str):
    res = ops.mxfp4_qdq_fwd(x.cuda(), block=32, scale_mode=mode, rowwise=True, emit_values=False,
                            emit_codes=True, emit_mask=True, scales_layout=layout, check=True)
    torch.cuda.synchronize()
    ora = O.qdq_rowwise(oracle_in(x), 32, 6.0, MODES[mode])
    exp_s = O.mma_scale_layout(ora["scales"]).reshape(-1) if layout == "mma" else ora["scales"]
    return res, ora, exp_s


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("layout", ["rowmajor", "mma"])
def test_every_bf16_value_codes_without_values(mode, layout):
    """The same sweep through the codes-only producer (no dequantised
    values: packed codes, scales, masks)."""
    xb = bf16_sweep_block32().reshape(-1, 256)  # 8 blocks per row
    x = torch.from_numpy(xb.view(np.int16).copy()).view(torch.bfloat16)
    res, ora, exp_s = codes_only(x, mode, layout)
    assert res.y_row is None
    assert np.array_equal(np_bits(res.codes_row), ora["codes"]), "codes"
    assert np.array_equal(np_bits(res.mask_row), ora["mask"]), "mask"
    assert np.array_equal(np_bits(res.scales_row).reshape(exp_s.shape), exp_s), "scales"


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("layout", ["rowmajor", "mma"])
@pytest.mark.parametrize("shape", [(300, 1024), (37, 4096), (1, 32), (129, 96), (64, 1000), (5, 999)])
def test_rowwise_codes_without_values(mode, layout, shape):
    """Codes, scales and masks without dequantised values on mixed inputs
    (specials included): the streaming producer where cols % 32 == 0, the
    staged and scalar kernels elsewhere."""
    x = W.mixed(*shape, seed=57 + shape[0])
    res, ora, exp_s = codes_only(x, mode, layout)
    assert np.array_equal(np_bits(res.codes_row), ora["codes"]), "codes"
    assert np.array_equal(np_bits(res.mask_row), ora["mask"]), "mask"
    assert np.array_equal(np_bits(res.scales_row).reshape(exp_s.shape), exp_s), "scales"


@pytest.mark.parametrize("grouped", [False, True])
def test_block128_many_tiles_per_cta(grouped):
    """Blocks of 128 in both directions on 9000 x 2048 (ragged last row block)
    and with 64 multinomial groups: every CTA of the persistent grid takes
    several tiles in turn, so the stage ring, both staging buffers and the
    per-parity column limits wrap many times."""
    rows, cols = 9000, 2048
    counts = W.moe_group_counts(rows, groups=64, seed=12).tolist() if grouped else None
    x = W.mixed(rows, cols, seed=77)
    res, ora = run_both(x, block=128, mode="page", rowwise=True, colwise=True, counts=counts)
    check_dir(res, ora["row"], "row", cols, label="b128 many tiles")
    check_dir(res, ora["col"], "col", cols, label="b128 many tiles")


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_every_bf16_value_block128_both_directions(mode):
    """Every finite bf16 value, in the low and the high half of a 32-bit word
    and with both signs, as element under fixed block maxima and as block
    maximum, through the dual kernel with blocks of 128: once with the
    sweep laid along rows, once along columns (the transpose)."""
    allv = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rows = []
    for shift in (0, 2):
        blk = np.zeros((65536, 128), np.uint16)
        blk[:, 0] = allv
        blk[:, 33] = np.where((allv & 0x7F80) >= (shift << 7), allv - (shift << 7), allv)
        blk[:, 98] = allv ^ 0x8000
        blk[:, 5] = 0x3F80
        rows.append(blk)
    for mx in (0x40C0, 0x4090, 0x3F80, 0x40F8, 0x0010, 0x7F7F):
        blk = np.zeros((65536, 128), np.uint16)
        blk[:, 127] = mx
        blk[:, 7] = allv
        blk[:, 64] = allv ^ 0x8000
        rows.append(blk)
    xb = np.concatenate(rows)
    for arr in (xb, np.ascontiguousarray(xb.T)):
        x = torch.from_numpy(arr.view(np.int16).copy()).view(torch.bfloat16)
        res, ora = run_both(x, block=128, mode=mode, rowwise=True, colwise=True)
        check_dir(res, ora["row"], "row", arr.shape[1], label="bf16 sweep b128")
        check_dir(res, ora["col"], "col", arr.shape[1], label="bf16 sweep b128")
        del res, ora, x


def test_fp32_random_patterns():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, (4096, 256), dtype=np.uint64).astype(np.uint32)
    bits[:1024] &= 0x807FFFFF  # subnormal-heavy rows
    bits[1024:2048] = (bits[1024:2048] & 0x80FFFFFF) | 0x3F000000  # values near 0.5..2
    x = torch.from_numpy(bits.view(np.float32).copy())
    for mode in ("page", "floor"):
        res, ora = run_both(x, block=32, mode=mode, rowwise=True, colwise=True)
        check_dir(res, ora["row"], "row", 256, label="fp32 patterns")
        check_dir(res, ora["col"], "col", 256, label="fp32 patterns")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("direction", ["rowwise", "colwise"])
@pytest.mark.parametrize("shape", [(300, 1024), (37, 1000), (5, 999)])
def test_ste_backward(dtype, direction, shape):
    x = W.mixed(*shape, dtype=dtype, seed=11)
    g = W.mixed(*shape, dtype=dtype, seed=12, specials=False)
    counts = [shape[0] // 3, 0, shape[0] - shape[0] // 3] if direction == "colwise" else None
    ends = None if counts is None else np.cumsum(counts)
    gl = None if counts is None else torch.tensor(counts, dtype=torch.int64, device="cuda")
    xd, gd = x.cuda(), g.cuda()
    xo, go = oracle_in(x), oracle_in(g)
    if direction == "rowwise":
        ora = O.qdq_rowwise(xo, 32, 6.0, O.SCALE_PAGE)
    else:
        ora = O.qdq_colwise(xo, 32, 6.0, O.SCALE_PAGE, ends=ends)
    exp = ora_bits(O.ste_bwd(go, ora["mask"], True))
    # 1) forward writes the mask, backward reads it
    res = ops.mxfp4_qdq_fwd(xd, rowwise=direction == "rowwise", colwise=direction == "colwise",
                            group_list=gl, group_list_type=1, emit_mask=True)
    m = res.mask_row if direction == "rowwise" else res.mask_col
    gi = ops.mxfp4_ste_bwd(gd, saved_mask=m, clip_grad=True)
    assert np.array_equal(np_bits(gi), exp)
    # 2) saved-free: recompute the mask from x
    gi = ops.mxfp4_ste_bwd(gd, x=xd, clip_grad=True, direction=direction, group_list=gl, group_list_type=1)
    assert np.array_equal(np_bits(gi), exp)
    # 3) fused forward + backward in one pass
    res, gi = ops.mxfp4_qdq_fwd_bwd(xd, gd, grad_direction=direction, rowwise=True, colwise=True,
                                    group_list=gl, group_list_type=1, emit_codes=True, emit_mask=True)
    assert np.array_equal(np_bits(gi), exp)
    check_dir(res, ora, "row" if direction == "rowwise" else "col", shape[1], label="fused")
    # 4) plain STE is the identity
    gi = ops.mxfp4_ste_bwd(gd, clip_grad=False)
    assert np.array_equal(np_bits(gi), np_bits(g))


@pytest.mark.parametrize("mode,sf", [("page", 6.0), ("page", 1.0), ("floor", 6.0)])
@pytest.mark.parametrize("shape", [(96, 2048), (33, 4096)])
def test_ste_recompute_rowwise_streaming(mode, sf, shape):
    """Saved-free row-wise STE on the streaming path (bf16, block 32, cols % 32
    == 0): special values, both scale rules, several scale factors."""
    x = W.mixed(*shape, dtype=torch.bfloat16, seed=21)
    g = W.mixed(*shape, dtype=torch.bfloat16, seed=22, specials=False)
    ora = O.qdq_rowwise(oracle_in(x), 32, sf, O.SCALE_PAGE if mode == "page" else O.SCALE_FLOOR)
    exp = ora_bits(O.ste_bwd(oracle_in(g), ora["mask"], True))
    gi = ops.mxfp4_ste_bwd(g.cuda(), x=x.cuda(), clip_grad=True, direction="rowwise", scale_factor=sf,
                           scale_mode=mode)
    assert np.array_equal(np_bits(gi), exp)


def test_invalid_group_list_writes_nothing_and_reports():
    x = W.mixed(100, 128, seed=13).cuda()
    for gl, t in (([50, 40, 60], 0), ([50, 60, 90], 0), ([50, -10, 60], 1), ([-1, 100], 0)):
        r = ops.alloc_outputs(x, block=32, rowwise=False, colwise=True, num_groups=len(gl), emit_codes=True,
                              emit_mask=True, with_status=True)
        for t_ in (r.y_col, r.codes_col, r.scales_col, r.mask_col):
            t_.view(torch.uint8).fill_(0xA5)
        glt = torch.tensor(gl, dtype=torch.int64, device="cuda")
        with pytest.raises(MXFP4ArgumentError):
            ops.mxfp4_qdq_fwd(x, rowwise=False, colwise=True, group_list=glt, group_list_type=t, out=r,
                              check=True)
        for t_ in (r.y_col, r.codes_col, r.scales_col, r.mask_col):
            assert bool((t_.view(torch.uint8) == 0xA5).all())


def test_empty_inputs():
    for shape in ((0, 64), (16, 0)):
        x = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        r = ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True, emit_codes=True, emit_mask=True)
        assert r.y_row.shape == shape
    with pytest.raises(ValueError):
        ops.mxfp4_qdq_fwd(torch.tensor(1.0, device="cuda"))


def test_cuda_graph_capture_and_replay():
    """The forward (dual, grouped, all outputs) and the STE backward capture
    into one CUDA graph: no host synchronisation or allocation on the path.
    Replays on new inputs copied into the captured buffers give the same
    bytes as eager calls."""
    rows, cols, counts = 640, 768, [100, 0, 37, 250, 253]
    gl = torch.tensor(np.cumsum(counts), dtype=torch.int64, device="cuda")
    xs = [W.mixed(rows, cols, seed=71 + i, specials=False) for i in range(3)]
    gs = [torch.randn(rows, cols, generator=torch.Generator().manual_seed(81 + i)).to(torch.bfloat16)
          for i in range(3)]
    xd, gd = xs[0].cuda(), gs[0].cuda()
    r = ops.alloc_outputs(xd, block=32, rowwise=True, colwise=True, num_groups=len(counts), emit_codes=True,
                          emit_mask=True, with_status=True)
    gi = torch.empty_like(gd)

    def step():
        ops.mxfp4_qdq_fwd(xd, rowwise=True, colwise=True, group_list=gl, emit_codes=True, emit_mask=True, out=r,
                          check=False)
        ops.mxfp4_ste_bwd(gd, saved_mask=r.mask_row, clip_grad=True, out=gi)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside the capture (kernel attributes, tensor maps)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    names = ("y_row", "y_col", "codes_row", "scales_row", "mask_row", "codes_col", "scales_col", "mask_col")
    for i in (1, 2, 0):
        xd.copy_(xs[i].cuda())
        gd.copy_(gs[i].cuda())
        graph.replay()
        torch.cuda.synchronize()
        got = {n: getattr(r, n).clone() for n in names}
        got_g = gi.clone()
        step()
        torch.cuda.synchronize()
        for n in names:
            assert torch.equal(got[n], getattr(r, n)), f"replay {i}: {n}"
        assert torch.equal(got_g.view(torch.int16), gi.view(torch.int16)), f"replay {i}: grad_in"
        assert int(r.status.item()) == 0
    ora = O.qdq_rowwise(oracle_in(xs[0]), 32, 6.0, O.SCALE_PAGE)
    check_dir(r, ora, "row", cols, label="graph replay")
    del graph
