"""GPU parity of the MXFP8 element format (E4M3 codes, E8M0 scale per 32)
against the CPU oracle, byte for byte: values, one-byte codes, scales and
saturation masks, row-wise (streaming and scalar kernels), column-wise with
group restarts, both directions, the STE backward, the MMA scale layout, and a
real MXFP8 block-scaled GEMM on the codes and scales."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import MXFP4ArgumentError, ops, workloads as W

pytestmark = pytest.mark.gpu


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


def check(res, ora, d, label=""):
    y, codes, scales, mask = (getattr(res, f"{k}_{d}") for k in ("y", "codes", "scales", "mask"))
    if y is not None:
        g, e = np_bits(y), ora_bits(ora["y"])
        bad = np.argwhere(g != e)
        assert bad.size == 0, f"{label} y_{d}: {len(bad)} mismatches, first {bad[:3].tolist()}"
    if codes is not None:
        g = np_bits(codes)
        bad = np.argwhere(g != ora["codes"])
        assert bad.size == 0, f"{label} codes_{d}: {len(bad)} mismatches, first {bad[:3].tolist()}"
    if scales is not None:
        s = ora["scales"].shape[0]
        assert np.array_equal(np_bits(scales)[:s], ora["scales"]), f"{label} scales_{d}"
    if mask is not None:
        assert np.array_equal(np_bits(mask), ora["mask"]), f"{label} mask_{d}"


def run(x, rowwise=True, colwise=False, counts=None, **kw):
    xd = x.cuda()
    gl, ends = None, None
    if counts is not None:
        ends = np.cumsum(np.asarray(counts, np.int64))
        gl = torch.tensor(ends, dtype=torch.int64, device="cuda")
    res = ops.mxfp4_qdq_fwd(xd, block=32, scale_mode="floor", rowwise=rowwise, colwise=colwise, group_list=gl,
                            emit_codes=True, emit_mask=True, check=True, elem_format="e4m3", **kw)
    torch.cuda.synchronize()
    xo = oracle_in(x)
    out = {}
    if rowwise:
        out["row"] = O.qdq8_rowwise(xo)
    if colwise:
        out["col"] = O.qdq8_colwise(xo, ends)
    return res, out


SHAPES = [(300, 1024), (64, 4096), (37, 1000), (129, 136), (5, 999), (2, 8), (1, 32)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", SHAPES)
def test_mxfp8_rowwise(dtype, shape):
    x = W.mixed(*shape, dtype=dtype, seed=200 + shape[0])
    res, ora = run(x)
    check(res, ora["row"], "row", f"{shape}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", SHAPES)
def test_mxfp8_colwise_and_dual(dtype, shape):
    x = W.mixed(*shape, dtype=dtype, seed=300 + shape[0])
    res, ora = run(x, rowwise=False, colwise=True)
    check(res, ora["col"], "col", f"col {shape}")
    res, ora = run(x, rowwise=True, colwise=True)
    check(res, ora["row"], "row", f"dual {shape}")
    check(res, ora["col"], "col", f"dual {shape}")


@pytest.mark.parametrize("counts", [[0, 45, 32, 0, 1, 70, 0], [31, 33, 64, 128, 44], [300]])
@pytest.mark.parametrize("cols", [256, 200, 99])
def test_mxfp8_grouped(counts, cols):
    x = W.mixed(sum(counts), cols, seed=400 + cols)
    res, ora = run(x, rowwise=True, colwise=True, counts=counts)
    check(res, ora["row"], "row", "grouped")
    check(res, ora["col"], "col", "grouped")
    assert int(res.status.item()) == 0


@pytest.mark.parametrize("cols", [256, 33])
def test_mxfp8_every_bf16_value(cols):
    """Every finite bf16 value as block maximum and as element under fixed
    maxima; 256 columns run the streaming kernel, 33 the scalar one."""
    allv = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rows = []
    for shift in (0, 2):
        blk = np.zeros((65536, 32), np.uint16)
        blk[:, 0] = allv
        blk[:, 1] = np.where((allv & 0x7F80) >= (shift << 7), allv - (shift << 7), allv)
        blk[:, 2] = allv ^ 0x8000
        rows.append(blk)
    for mx in (0x43E0, 0x4380, 0x3F80, 0x0010, 0x7F7F, 0x0C00):
        blk = np.zeros((65536, 32), np.uint16)
        blk[:, 0] = mx
        blk[:, 7] = allv
        rows.append(blk)
    xb = np.concatenate(rows)
    if cols == 256:
        xb = xb.reshape(-1, 256)
    else:
        xb = np.concatenate([xb, np.zeros((xb.shape[0], 1), np.uint16)], axis=1)
    x = torch.from_numpy(xb.view(np.int16).copy()).view(torch.bfloat16)
    res, ora = run(x)
    check(res, ora["row"], "row", f"sweep {cols}")


# bf16 inputs with cols % 32 == 0 run the staged kernel in the column-wise
# and dual calls: partial column tiles (warps past the last column), ragged
# and group-tail row blocks, many tiles per CTA (the stage ring wraps)
@pytest.mark.parametrize("shape,counts", [((96, 288), None), ((1000, 800), None), ((33, 32), None),
                                          ((700, 1312), [0, 45, 320, 0, 1, 300, 34]),
                                          ((16384, 2048), "moe")])
def test_mxfp8_staged_shapes(shape, counts):
    rows, cols = shape
    if counts == "moe":
        counts = W.moe_group_counts(rows, groups=64, seed=8).tolist()
    x = W.mixed(rows, cols, seed=500 + cols)
    res, ora = run(x, rowwise=True, colwise=True, counts=counts)
    check(res, ora["row"], "row", f"dual {shape}")
    check(res, ora["col"], "col", f"dual {shape}")
    res, ora = run(x, rowwise=False, colwise=True, counts=counts)
    check(res, ora["col"], "col", f"col {shape}")


@pytest.mark.parametrize("counts", [None, [17, 47]])
def test_mxfp8_every_bf16_value_along_columns(counts):
    """The sweep of test_mxfp8_every_bf16_value laid along columns (each
    32-element block is one column of 32 rows), through the staged kernel's
    column pass, in both directions; with groups the blocks are cut at 17
    rows."""
    allv = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blocks = []
    for shift in (0, 2):
        blk = np.zeros((65536, 32), np.uint16)
        blk[:, 0] = allv
        blk[:, 1] = np.where((allv & 0x7F80) >= (shift << 7), allv - (shift << 7), allv)
        blk[:, 2] = allv ^ 0x8000
        blocks.append(blk)
    for mx in (0x43E0, 0x4380, 0x3F80, 0x0010, 0x7F7F, 0x0C00):
        blk = np.zeros((65536, 32), np.uint16)
        blk[:, 0] = mx
        blk[:, 7] = allv
        blocks.append(blk)
    xb = np.concatenate(blocks)  # (524288, 32): one block per row
    half = xb.shape[0] // 2
    xb = np.concatenate([xb[:half].T, xb[half:].T])  # (64, 262144): one block per column
    x = torch.from_numpy(np.ascontiguousarray(xb).view(np.int16)).view(torch.bfloat16)
    res, ora = run(x, rowwise=True, colwise=True, counts=counts)
    check(res, ora["col"], "col", "column sweep")
    check(res, ora["row"], "row", "column sweep")


@pytest.mark.parametrize("direction", ["rowwise", "colwise"])
def test_mxfp8_ste(direction):
    x = W.mixed(96, 512, seed=17)
    g = torch.randn(96, 512, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    xo = oracle_in(x)
    ora = O.qdq8_rowwise(xo) if direction == "rowwise" else O.qdq8_colwise(xo)
    exp = O.ste_bwd(oracle_in(g), ora["mask"], True)
    res, _ = run(x, rowwise=direction == "rowwise", colwise=direction == "colwise")
    mask = res.mask_row if direction == "rowwise" else res.mask_col
    gi = ops.mxfp4_ste_bwd(g.cuda(), saved_mask=mask, clip_grad=True)
    assert np.array_equal(np_bits(gi), exp)
    gi2 = ops.mxfp4_ste_bwd(g.cuda(), x=x.cuda(), clip_grad=True, scale_mode="floor", direction=direction,
                            elem_format="e4m3")
    assert np.array_equal(np_bits(gi2), exp)
    r3, gi3 = ops.mxfp4_qdq_fwd_bwd(x.cuda(), g.cuda(), grad_direction=direction, scale_mode="floor",
                                    rowwise=direction == "rowwise", colwise=direction == "colwise",
                                    elem_format="e4m3")
    torch.cuda.synchronize()
    assert np.array_equal(np_bits(gi3), exp)


def test_mxfp8_mma_scale_layout():
    x = W.mixed(300, 1024, seed=23)
    res = ops.mxfp4_qdq_fwd(x.cuda(), block=32, scale_mode="floor", rowwise=True, emit_codes=True,
                            emit_mask=True, scales_layout="mma", elem_format="e4m3")
    torch.cuda.synchronize()
    ora = O.qdq8_rowwise(oracle_in(x))
    assert np.array_equal(np_bits(res.scales_row), O.mma_scale_layout(ora["scales"]))
    assert np.array_equal(np_bits(res.codes_row), ora["codes"])


@pytest.mark.parametrize("shape,counts", [((300, 1024), None), ((261, 288), [100, 0, 61, 100]),
                                          ((4096, 2048), "moe")])
def test_mxfp8_dual_mma_scale_layout(shape, counts):
    """Both directions with the row-wise scales in the MMA layout (the staged
    kernel's SMMA form): the scales equal the oracle's placed by its layout
    helper, unaligned by one byte too, and every other output is unchanged."""
    rows, cols = shape
    if counts == "moe":
        counts = W.moe_group_counts(rows, groups=32, seed=14).tolist()
    x = W.mixed(rows, cols, seed=60 + rows)
    xd = x.cuda()
    xo = oracle_in(x)
    ora = O.qdq8_rowwise(xo)
    for soff in (0, 1):
        r = ops.alloc_outputs(xd, block=32, rowwise=True, colwise=True,
                              num_groups=0 if counts is None else len(counts), emit_codes=True, emit_mask=True,
                              with_status=True, scales_layout="mma", elem_format="e4m3")
        n = r.scales_row.numel()
        r.scales_row = torch.zeros((n + soff,), dtype=torch.uint8, device=xd.device)[soff:]
        gl = None if counts is None else torch.tensor(counts, dtype=torch.int64, device=xd.device)
        ops.mxfp4_qdq_fwd(xd, block=32, scale_mode="floor", rowwise=True, colwise=True, group_list=gl,
                          group_list_type=1, emit_codes=True, emit_mask=True, out=r, check=True,
                          elem_format="e4m3")
        torch.cuda.synchronize()
        got = r.scales_row.cpu().numpy()
        exp = O.mma_scale_layout(ora["scales"])
        bad = np.flatnonzero(got != exp)
        assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:4].tolist()}"
        r.scales_row = None
        check(r, ora, "row", f"mma {shape}")
        ends = None if counts is None else np.cumsum(np.asarray(counts, np.int64))
        check(r, O.qdq8_colwise(xo, ends), "col", f"mma {shape}")


def test_mxfp8_argument_errors():
    x = torch.randn(64, 64, device="cuda").to(torch.bfloat16)
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_qdq_fwd(x, block=32, scale_mode="page", elem_format="e4m3")
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_qdq_fwd(x, block=128, scale_mode="floor", elem_format="e4m3")
    with pytest.raises(ValueError):
        ops.mxfp4_qdq_fwd(x, block=32, scale_mode="floor", elem_format="e5m2")


@pytest.mark.parametrize("mnk", [(256, 384, 2048), (192, 256, 1024)])
def test_mxfp8_operands_in_a_real_gemm(mnk):
    """E4M3 codes and MMA-layout E8M0 scales fed to torch's MXFP8 block-scaled
    GEMM give the product of the fake-quantised matrices (oracle values in
    float64), within the bf16 output rounding plus fp32 accumulation."""
    from torch.nn.functional import ScalingType, SwizzleType, scaled_mm
    M, N, K = mnk
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16)
    w = torch.randn(N, K, generator=torch.Generator().manual_seed(N + 7)).to(torch.bfloat16)
    rx = ops.mxfp4_qdq_fwd(x.cuda(), block=32, scale_mode="floor", rowwise=True, emit_values=False,
                           emit_codes=True, scales_layout="mma", elem_format="e4m3")
    rw = ops.mxfp4_qdq_fwd(w.cuda(), block=32, scale_mode="floor", rowwise=True, emit_values=False,
                           emit_codes=True, scales_layout="mma", elem_format="e4m3")
    out = scaled_mm(rx.codes_row.view(torch.float8_e4m3fn), rw.codes_row.view(torch.float8_e4m3fn).t(),
                    rx.scales_row.view(torch.float8_e8m0fnu), ScalingType.BlockWise1x32,
                    rw.scales_row.view(torch.float8_e8m0fnu), ScalingType.BlockWise1x32,
                    swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                    output_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    yx = O.bf16_to_f32(O.qdq8_rowwise(oracle_in(x))["y"]).astype(np.float64)
    yw = O.bf16_to_f32(O.qdq8_rowwise(oracle_in(w))["y"]).astype(np.float64)
    ref = yx @ yw.T
    mag = np.abs(yx) @ np.abs(yw).T
    err = np.abs(out.float().cpu().numpy().astype(np.float64) - ref)
    bound = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * mag
    assert np.all(err <= bound), f"max err/bound {float((err / bound).max()):.3f}"
