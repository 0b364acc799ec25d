"""GPU parity of the column-wise real-quantisation operand (col_layout
"mma", include/mxfp4.h MXFP4_COLS_MMA): the K-major codes and MMA-layout
scales of a GEMM that contracts over the rows group by group, byte for byte
against the oracle's column-wise result placed by the oracle's layout helper
(oracle.colwise_operand_layout, pinned by hand offsets), and fed to a real
block-scaled FP4 GEMM per group (the weight-gradient direction of MindSpore
hyper-parallel fake_w4a8_gmm_func.py, FakeW4A8GroupedLinear._select_operands,
layout "TN")."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import MXFP4ArgumentError, ops, workloads as W

pytestmark = pytest.mark.gpu

MODES = {"page": O.SCALE_PAGE, "floor": O.SCALE_FLOOR}


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


CASES = [
    (300, 256, None),
    (261, 1000, [100, 0, 61, 100]),
    (1000, 130, [0, 500, 1, 499]),
    (64, 6, [64]),
    (129, 7, [5, 124]),
    (40, 64, [0, 0, 40, 0]),
]


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("case", CASES)
def test_colwise_operand_bytes(mode, case):
    rows, cols, counts = case
    x = W.mixed(rows, cols, seed=90 + rows + cols)
    ends = None if counts is None else np.cumsum(np.asarray(counts, np.int64))
    ora = O.qdq_colwise(u16(x), 32, 6.0, MODES[mode], ends=ends)
    e = np.array([rows]) if ends is None else ends
    k = O.colwise_operand_k(e)
    for k_alloc, host_list in ((None, True), (k + 256, False)):
        gl = None if counts is None else (list(counts) if host_list else
                                          torch.tensor(counts, dtype=torch.int64, device="cuda"))
        codes, scales, ka = ops.mxfp4_colwise_mma_operand(x.cuda(), group_list=gl, group_list_type=1,
                                                          scale_mode=mode, k_alloc=k_alloc)
        assert ka == (k if k_alloc is None else k_alloc)
        exp_c, exp_s = O.colwise_operand_layout(ora["codes"], ora["scales"], e, cols, k_alloc=ka)
        got_c = codes.view(torch.uint8).cpu().numpy()
        got_s = scales.view(torch.uint8).cpu().numpy()
        assert got_c.shape == exp_c.shape
        bad = np.argwhere(got_c != exp_c)
        assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:3].tolist()}"
        bad = np.flatnonzero(got_s != exp_s)
        assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("grouped", [False, True])
def test_colwise_operand_many_tiles(grouped):
    """cols % 32 == 0 runs the TMA-staged producer: 9000 x 2048 with 64
    multinomial groups (or none), several tiles per CTA, so its stage ring
    wraps, tails and padding block pairs of every kind occur."""
    rows, cols = 9000, 2048
    counts = W.moe_group_counts(rows, groups=64, seed=13).tolist() if grouped else None
    x = W.mixed(rows, cols, seed=31)
    ends = np.array([rows]) if counts is None else np.cumsum(np.asarray(counts, np.int64))
    ora = O.qdq_colwise(u16(x), 32, 6.0, O.SCALE_PAGE, ends=None if counts is None else ends)
    codes, scales, ka = ops.mxfp4_colwise_mma_operand(x.cuda(), group_list=counts, group_list_type=1)
    exp_c, exp_s = O.colwise_operand_layout(ora["codes"], ora["scales"], ends, cols, k_alloc=ka)
    got_c = codes.view(torch.uint8).cpu().numpy()
    got_s = scales.view(torch.uint8).cpu().numpy()
    bad = np.argwhere(got_c != exp_c)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:3].tolist()}"
    bad = np.flatnonzero(got_s != exp_s)
    assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:4].tolist()}"


def test_dual_call_with_operand_layout():
    """Row-wise outputs, column-wise values and masks, and the column-wise
    operand from one call: each equals the oracle."""
    rows, cols, counts = 300, 512, [100, 0, 37, 163]
    x = W.mixed(rows, cols, seed=5)
    ends = np.cumsum(counts)
    gl = torch.tensor(counts, dtype=torch.int64, device="cuda")
    r = ops.mxfp4_qdq_fwd(x.cuda(), rowwise=True, colwise=True, group_list=gl, group_list_type=1, emit_codes=True,
                          emit_mask=True, col_layout="mma")
    xo = u16(x)
    orow = O.qdq_rowwise(xo, 32, 6.0, O.SCALE_PAGE)
    ocol = O.qdq_colwise(xo, 32, 6.0, O.SCALE_PAGE, ends=ends)
    assert np.array_equal(u16(r.y_row), orow["y"]) and np.array_equal(r.codes_row.cpu().numpy(), orow["codes"])
    assert np.array_equal(r.scales_row.cpu().numpy(), orow["scales"])
    assert np.array_equal(r.mask_row.cpu().numpy(), orow["mask"])
    assert np.array_equal(u16(r.y_col), ocol["y"]) and np.array_equal(r.mask_col.cpu().numpy(), ocol["mask"])
    exp_c, exp_s = O.colwise_operand_layout(ocol["codes"], ocol["scales"], ends, cols, k_alloc=r.k_alloc)
    assert np.array_equal(r.codes_col.cpu().numpy(), exp_c)
    assert np.array_equal(r.scales_col.cpu().numpy(), exp_s)


def test_k_alloc_too_small_for_the_groups_is_reported():
    rows, cols = 300, 64
    x = W.mixed(rows, cols, seed=8).cuda()
    gl = torch.tensor([1, 1, 1, 297], dtype=torch.int64, device="cuda")  # needs 4 * 128 + 256 = 768 K slots
    r = ops.alloc_outputs(x, block=32, rowwise=False, colwise=True, num_groups=4, emit_values=False, emit_codes=True,
                          with_status=True, col_layout="mma", k_alloc=512)
    r.codes_col.fill_(0xA5)
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_qdq_fwd(x, rowwise=False, colwise=True, group_list=gl, group_list_type=1, emit_values=False,
                          out=r, check=True)
    assert bool((r.codes_col == 0xA5).all())
    with pytest.raises(MXFP4ArgumentError):  # not a multiple of 128: rejected on the host
        ops.mxfp4_colwise_mma_operand(x, k_alloc=320)
    with pytest.raises(MXFP4ArgumentError):  # too small without groups: rejected on the host
        ops.mxfp4_colwise_mma_operand(x, k_alloc=256)


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_operand_in_a_real_grouped_fp4_gemm(mode):
    """Per group g, torch's block-scaled FP4 GEMM (MXFP4: E2M1 data, E8M0
    scales per 32 along K, 128 x 4 atoms) on the group's slice of the
    column-wise operands of X and dY gives X_g^T dY_g of the fake-quantised
    (column-wise, group-restarting) matrices. Reference: the oracle's
    dequantised values multiplied in float64; bound: bf16 output rounding plus
    fp32 accumulation."""
    from torch.nn.functional import ScalingType, SwizzleType, scaled_mm
    counts = [200, 0, 77, 328, 5]
    rows, cx, cy = sum(counts), 256, 384
    ends = np.cumsum(counts)
    x = torch.randn(rows, cx, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    dy = (torch.randn(rows, cy, generator=torch.Generator().manual_seed(2)) * 1e-3).to(torch.bfloat16)
    ca, sa, ka = ops.mxfp4_colwise_mma_operand(x.cuda(), group_list=counts, group_list_type=1, scale_mode=mode)
    cb, sb, kb = ops.mxfp4_colwise_mma_operand(dy.cuda(), group_list=counts, group_list_type=1, scale_mode=mode)
    assert ka == kb
    qx = O.bf16_to_f32(O.qdq_colwise(u16(x), 32, 6.0, MODES[mode], ends=ends)["y"]).astype(np.float64)
    qy = O.bf16_to_f32(O.qdq_colwise(u16(dy), 32, 6.0, MODES[mode], ends=ends)["y"]).astype(np.float64)
    sa_at = sa.view(torch.uint8).view(cx // 128, ka // 128, 512)
    sb_at = sb.view(torch.uint8).view(cy // 128, ka // 128, 512)
    k0, start = 0, 0
    for n in counts:
        kpad = -(-n // 128) * 128
        if n == 0:
            continue
        a = ca.view(torch.uint8)[:, k0 // 2:(k0 + kpad) // 2].contiguous().view(torch.float4_e2m1fn_x2)
        b = cb.view(torch.uint8)[:, k0 // 2:(k0 + kpad) // 2].contiguous().view(torch.float4_e2m1fn_x2)
        s_a = sa_at[:, k0 // 128:(k0 + kpad) // 128].contiguous().view(-1).view(torch.float8_e8m0fnu)
        s_b = sb_at[:, k0 // 128:(k0 + kpad) // 128].contiguous().view(-1).view(torch.float8_e8m0fnu)
        out = scaled_mm(a, b.t(), s_a, ScalingType.BlockWise1x32, s_b, ScalingType.BlockWise1x32,
                        swizzle_a=SwizzleType.SWIZZLE_32_4_4, swizzle_b=SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        xg, yg = qx[start:start + n], qy[start:start + n]
        ref = xg.T @ yg
        mag = np.abs(xg).T @ np.abs(yg)
        err = np.abs(out.float().cpu().numpy().astype(np.float64) - ref)
        bound = 2.0 ** -8 * np.abs(ref) + kpad * 2.0 ** -23 * mag + 1e-30
        assert np.all(err <= bound), f"group of {n}: max err/bound {float((err / bound).max()):.3f}"
        k0 += kpad
        start += n
