"""GPU parity at the workloads' full sizes: every output element compared.

The five workloads of the benchmark suite at their stated shapes (the tiny
QAT linear is covered in test_gpu_qat.py), in both scale rules, launched the
way the benchmark launches them, and compared byte for byte with the oracle
over the whole tensor (the oracle runs on row or column chunks on several
host threads; tests/oracle_par.py). Tolerance: 0 ULP, as everywhere.

The training-step workload's injected blocks (all-zero blocks every 4096th
block, the subnormal block in row 3, the +inf / -inf / NaN blocks in row 7)
are part of the full compare and are also asserted explicitly, so that a
workload that lost them would fail here.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import ops, workloads as W
from tests import oracle_par as OP

pytestmark = pytest.mark.gpu

MODES = {"page": O.SCALE_PAGE, "floor": O.SCALE_FLOOR}


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def same(got: torch.Tensor, exp: np.ndarray, label: str) -> None:
    g = bits(got)
    if g.shape != exp.shape:
        g = g.reshape(exp.shape)
    if np.array_equal(g, exp):
        return
    bad = np.argwhere(g != exp)
    i = tuple(bad[0])
    raise AssertionError(f"{label}: {len(bad)} of {exp.size} differ; first at {list(i)}: "
                         f"gpu {int(g[i]):#x} oracle {int(exp[i]):#x}")


def check(res: ops.QDQResult, ora: dict, d: str, label: str) -> None:
    for k in ("y", "codes", "scales", "mask"):
        t = getattr(res, f"{k}_{d}")
        if t is None:
            continue
        e = ora[k]
        if k == "scales" and d == "col":
            t = t[: e.shape[0]]
        same(t, e, f"{label} {k}_{d}")


@pytest.fixture(autouse=True)
def _free_device_memory():
    torch.cuda.empty_cache()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_activation_rowwise_full(mode):
    """bf16 [8192, 4096], N(0,1) with 20 outlier channels x50: row-wise block
    32 with values, codes and scales (the streaming kernel), then with the
    saturation mask as well."""
    x = W.act_rowwise()
    xd = x.cuda()
    ora = OP.qdq_rowwise(bits(x), 32, 6.0, MODES[mode])
    r = ops.mxfp4_qdq_fwd(xd, scale_mode=mode, emit_codes=True)
    check(r, ora, "row", f"act {mode}")
    r = ops.mxfp4_qdq_fwd(xd, scale_mode=mode, emit_codes=True, emit_mask=True)
    check(r, ora, "row", f"act+mask {mode}")


@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("mode", ["page", "floor"])
def test_weight_dual_full(mode, block):
    """bf16 [14336, 4096] ~ N(0, 0.02^2): both directions from one read, every
    output, blocks of 32 and of 128."""
    x = W.weight_dual()
    xd = x.cuda()
    r = ops.mxfp4_qdq_fwd(xd, block=block, scale_mode=mode, rowwise=True, colwise=True, emit_codes=True,
                          emit_mask=True)
    xb = bits(x)
    check(r, OP.qdq_rowwise(xb, block, 6.0, MODES[mode]), "row", f"weight b{block} {mode}")
    check(r, OP.qdq_colwise(xb, block, 6.0, MODES[mode]), "col", f"weight b{block} {mode}")


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_training_step_full(mode):
    """bf16 x [16384, 4096] = 0.5 Student-t(4), grad_out ~ N(0, 1e-6): the
    forward with codes, scales and the saved mask, the clipped STE from the
    saved mask and recomputed from x (saved-free), and the fused forward +
    backward, all against the oracle; the injected special blocks included."""
    x, g = W.train_step()
    xd, gd = x.cuda(), g.cuda()
    xb, gb = bits(x), bits(g)
    ora = OP.qdq_rowwise(xb, 32, 6.0, MODES[mode])
    exp_g = OP.ste_bwd(gb, ora["mask"], True)

    # the injections are in the input, and the oracle treats them as the
    # pages' arithmetic says
    nb = x.shape[1] // 32
    assert all(int(ora["scales"][7, b]) == 0xFF for b in (3, 4, 5))
    assert np.all(ora["y"][7, 3 * 32: 6 * 32] == 0x7FC0)
    assert not ora["mask"][7, 12:24].any()
    sub = xb[3, 32:64]
    assert int((sub & 0x7FFF).max()) == W.SUBNORMAL_2_M130 and not (sub & 0x7F80).any()
    assert int(ora["scales"][3, 1]) == (97 if mode == "page" else 0)
    zero_blocks = np.arange(0, x.shape[0] * nb, 4096)
    zr, zb = zero_blocks // nb, zero_blocks % nb
    assert not xb.reshape(-1, 32)[zero_blocks].any()
    assert np.all(ora["scales"][zr, zb] == (97 if mode == "page" else 0))

    r = ops.mxfp4_qdq_fwd(xd, scale_mode=mode, emit_codes=True, emit_mask=True)
    check(r, ora, "row", f"train fwd {mode}")
    same(ops.mxfp4_ste_bwd(gd, saved_mask=r.mask_row, clip_grad=True), exp_g, f"train ste saved {mode}")
    same(ops.mxfp4_ste_bwd(gd, x=xd, clip_grad=True, scale_mode=mode), exp_g, f"train ste recompute {mode}")
    same(ops.mxfp4_ste_bwd(gd, saved_mask=r.mask_row, clip_grad=False), gb, f"train plain ste {mode}")
    rf, gf = ops.mxfp4_qdq_fwd_bwd(xd, gd, scale_mode=mode, emit_mask=True)
    same(rf.y_row, ora["y"], f"train fused y {mode}")
    same(rf.mask_row, ora["mask"], f"train fused mask {mode}")
    same(gf, exp_g, f"train fused grad {mode}")


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_moe_grouped_full(mode):
    """bf16 [65536, 7168] ~ N(0,1) with 256 multinomial groups (three empty):
    the benchmark step in full -- both directions with column-wise blocks
    restarting at every group, every output, then the clipped STE from the
    saved row-wise mask."""
    x, counts, offsets = W.moe_grouped()
    assert int((counts == 0).sum()) >= 3
    xd, gl = x.cuda(), offsets.cuda()
    r = ops.mxfp4_qdq_fwd(xd, scale_mode=mode, rowwise=True, colwise=True, group_list=gl, emit_codes=True,
                          emit_mask=True)
    xb = bits(x)
    ends = offsets.numpy()
    assert r.scales_col.shape[0] >= O.colwise_scale_rows(ends, 32)
    ora_r = OP.qdq_rowwise(xb, 32, 6.0, MODES[mode])
    check(r, ora_r, "row", f"moe {mode}")
    ora_c = OP.qdq_colwise(xb, 32, 6.0, MODES[mode], ends)
    check(r, ora_c, "col", f"moe {mode}")
    del ora_c
    g = W.train_step_grad(*x.shape)
    gi = ops.mxfp4_ste_bwd(g.cuda(), saved_mask=r.mask_row, clip_grad=True)
    same(gi, OP.ste_bwd(bits(g), ora_r["mask"], True), f"moe ste {mode}")


def test_bench_modes_full():
    """The other calls the benchmark times, on its full tensor (65536 x 7168):
    the real-quantisation producer (codes + MMA-layout scales, no values), the
    training step (row-wise forward with every output, saved-free STE), blocks
    of 128 in both directions, and MXFP8 row-wise and in both directions with
    the groups -- each compared in full."""
    x, counts, offsets = W.moe_grouped()
    xd, gl = x.cuda(), offsets.cuda()
    xb = bits(x)
    ends = offsets.numpy()
    ora = OP.qdq_rowwise(xb, 32, 6.0, O.SCALE_PAGE)
    codes, scales = ops.mxfp4_mma_operand(xd)
    same(codes.view(torch.uint8), ora["codes"], "producer codes")
    same(scales.view(torch.uint8), O.mma_scale_layout(ora["scales"]), "producer scales")
    del codes, scales
    r = ops.mxfp4_qdq_fwd(xd, emit_codes=True, emit_mask=True)
    check(r, ora, "row", "row-wise all outputs")
    g = W.train_step_grad(*x.shape)
    same(ops.mxfp4_ste_bwd(g.cuda(), x=xd, clip_grad=True), OP.ste_bwd(bits(g), ora["mask"], True),
         "saved-free ste")
    del r, ora, g
    r = ops.mxfp4_qdq_fwd(xd, block=128, rowwise=True, colwise=True, emit_codes=True, emit_mask=True)
    check(r, OP.qdq_rowwise(xb, 128, 6.0, O.SCALE_PAGE), "row", "b128")
    check(r, OP.qdq_colwise(xb, 128, 6.0, O.SCALE_PAGE), "col", "b128")
    del r
    r = ops.mxfp4_qdq_fwd(xd, block=32, scale_mode="floor", rowwise=True, colwise=True, group_list=gl,
                          emit_codes=True, emit_mask=True, elem_format="e4m3")
    check(r, OP.qdq8_rowwise(xb), "row", "mxfp8")
    check(r, OP.qdq8_colwise(xb, ends), "col", "mxfp8")
