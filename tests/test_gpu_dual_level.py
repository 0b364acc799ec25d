"""GPU parity of the dual-level MX quantisation kernel against the oracle.

Reading (sglang mxfp4_npu.py, NPUMXFP4DiffusionLinearMethod,
npu_dynamic_dual_level_mx_quant; the page gives the operator's results only):
fp32 level-0 scale s0 = amax0 / 6 per 512 elements of a row, level-1 MXFP4
QDQ (amct pull request 264, mxfp4_qat/fake_quant.py) of y = x / s0 with
blocks of 32, output code * 2^k1 * s0 in bf16. Every output (values, packed
codes, fp32 level-0 scales, E8M0 level-1 scales, saturation bits) is compared
byte for byte: 0 ULP.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import MXFP4ArgumentError, ops, workloads as W
from tests import oracle_par as OP

pytestmark = pytest.mark.gpu

MODES = {"page": O.SCALE_PAGE, "floor": O.SCALE_FLOOR}


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.numpy()


def same(got: torch.Tensor, exp: np.ndarray, label: str) -> None:
    g = bits(got)
    e = exp.view(np.uint32) if exp.dtype == np.float32 else exp
    if np.array_equal(g, e):
        return
    bad = np.argwhere(g != e)
    i = tuple(bad[0])
    raise AssertionError(f"{label}: {len(bad)} of {e.size} differ; first at {list(i)}: "
                         f"gpu {int(g[i]):#x} oracle {int(e[i]):#x}")


def check_all(r: ops.DualLevelResult, ora: dict, label: str) -> None:
    for k in ("y", "codes", "scales0", "scales1", "mask"):
        t = getattr(r, k)
        if t is not None:
            same(t, ora[k], f"{label} {k}")


def u16(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("rows,cols", [(64, 4096), (33, 1000), (7, 512), (1, 37), (5, 1001), (300, 7168),
                                       (2, 3), (129, 520)])
def test_dual_level_parity(mode, rows, cols):
    """Many units per warp, ragged level-0 and level-1 tails, odd widths (the
    general path), one-row and tiny tensors; mixed magnitudes, subnormals,
    zeros and +-inf / NaN blocks."""
    x = W.mixed(rows, cols, seed=rows * 7 + cols)
    r = ops.mxfp4_dual_level_qdq(x.cuda(), scale_mode=mode, emit_mask=True)
    torch.cuda.synchronize()
    check_all(r, O.dual_level_rowwise(u16(x), 512, 6.0, MODES[mode]), f"{rows}x{cols} {mode}")


@pytest.mark.parametrize("sf", [4.0, 0.75, 9.5, 2.0 ** -40, 1000.0])
def test_dual_level_scale_factors(sf):
    """The level-1 PAGE rule with other scale factors (some outside the range
    of the single-level fast paths)."""
    x = W.mixed(48, 2048, seed=5)
    r = ops.mxfp4_dual_level_qdq(x.cuda(), scale_mode="page", scale_factor=sf, emit_mask=True)
    torch.cuda.synchronize()
    check_all(r, O.dual_level_rowwise(u16(x), 512, sf, O.SCALE_PAGE), f"sf={sf}")


def every_value_rows(a0_bits: np.ndarray) -> np.ndarray:
    """Rows of 512: element 0 is the level-0 amax a0 itself, the other 511 run
    through every finite bf16 x with |x| <= a0 (both signs), so that each such
    x is quantised under each listed a0."""
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mag = allb & 0x7FFF
    fin = allb[mag < 0x7F80]
    out = []
    for a in a0_bits:
        xs = fin[(fin & 0x7FFF) <= a]
        n = -(-xs.size // 511)
        body = np.zeros(n * 511, np.uint16)
        body[: xs.size] = xs
        rows = np.concatenate([np.full((n, 1), a, np.uint16), body.reshape(n, 511)], axis=1)
        out.append(rows)
    return np.concatenate(out)


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_every_bf16_value_under_many_level0_scales(mode):
    """Every finite bf16 value as an element under every level-0 amax
    significand (exponent 0), and under amaxes at the extremes (the smallest
    subnormal, the smallest normal, 2^-120 * 1.5, 2^100, the largest bf16):
    exercises the corrected reciprocal product and the IEEE-division fallback
    (tiny elements, tiny level-0 scales)."""
    sig = (0x3F80 + np.arange(128)).astype(np.uint16)
    ext = np.array([0x0001, 0x0080, 0x03C0, 0x7180, 0x7F7F], np.uint16)
    x = every_value_rows(np.concatenate([sig, ext]))
    r = ops.mxfp4_dual_level_qdq(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda(),
                                 scale_mode=mode, emit_mask=True)
    torch.cuda.synchronize()
    check_all(r, OP.dual_level_rowwise(x, 512, 6.0, MODES[mode]), f"every value {mode}")


def test_dual_level_strided_input_and_output_subsets():
    """A strided row view (ld > cols, 16-byte aligned and not), and calls that
    ask for some outputs only."""
    base = W.mixed(40, 3072, seed=12)
    ora_full = O.dual_level_rowwise(u16(base[:, :2048].contiguous()), 512, 6.0, O.SCALE_FLOOR)
    xd = base.cuda()
    r = ops.mxfp4_dual_level_qdq(xd[:, :2048], scale_mode="floor", emit_mask=True)  # ld 3072, vector path
    torch.cuda.synchronize()
    check_all(r, ora_full, "ld 3072")
    off = ops.mxfp4_dual_level_qdq(xd[:, 1:2049], scale_mode="floor", emit_mask=True)  # misaligned start
    torch.cuda.synchronize()
    check_all(off, O.dual_level_rowwise(u16(base[:, 1:2049].contiguous()), 512, 6.0, O.SCALE_FLOOR), "offset 1")
    only = ops.mxfp4_dual_level_qdq(xd[:, :2048], scale_mode="floor", emit_values=False, emit_codes=True)
    torch.cuda.synchronize()
    assert only.y is None and only.mask is None
    check_all(only, ora_full, "codes + scales only")
    vals = ops.mxfp4_dual_level_qdq(xd[:, :2048], scale_mode="floor", emit_codes=False)
    torch.cuda.synchronize()
    check_all(vals, ora_full, "values + scales only")


def test_dual_level_clipped_ste_from_saved_mask():
    """The dual-level saturation mask drives the clipped STE backward through
    mxfp4_ste_bwd unchanged (amct pull request 264, _MXFP4FakeQuantSTE)."""
    x = W.mixed(96, 1536, seed=21, specials=False)
    g = torch.randn(96, 1536, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    r = ops.mxfp4_dual_level_qdq(x.cuda(), emit_mask=True)
    gi = ops.mxfp4_ste_bwd(g.cuda(), saved_mask=r.mask, clip_grad=True)
    torch.cuda.synchronize()
    ora = O.dual_level_rowwise(u16(x), 512, 6.0, O.SCALE_PAGE)
    same(gi, O.ste_bwd(u16(g), ora["mask"], True), "clipped STE grad")
    assert O.unpack_bits(ora["mask"], 1536).any()  # the case exercises the mask


def test_dual_level_empty_and_rejected():
    e = ops.mxfp4_dual_level_qdq(torch.empty((0, 512), dtype=torch.bfloat16, device="cuda"))
    assert e.y.shape == (0, 512) and e.scales0.shape == (0, 1)
    with pytest.raises(TypeError):
        ops.mxfp4_dual_level_qdq(torch.zeros((4, 512), device="cuda"))
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_dual_level_qdq(torch.zeros((4, 512), dtype=torch.bfloat16, device="cuda"), level0_block=256)
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_dual_level_qdq(torch.zeros((4, 512), dtype=torch.bfloat16, device="cuda"), level0_block=100)


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_dual_level_full_size(mode):
    """The benchmark's tensor, bf16 [65536, 7168] N(0,1) (470M elements),
    every output compared in full, launched as the benchmark launches it."""
    x = W.moe_grouped(65536, 7168, 256, 4)[0]
    r = ops.mxfp4_dual_level_qdq(x.cuda(), scale_mode=mode, emit_mask=True)
    torch.cuda.synchronize()
    check_all(r, OP.dual_level_rowwise(u16(x), 512, 6.0, MODES[mode]), f"full size {mode}")


def test_dual_level_into_caller_buffers():
    """Outputs written into caller-provided tensors (the `out` argument); a
    buffer of the wrong shape or dtype is rejected before any launch."""
    x = W.mixed(20, 1024, seed=31, specials=False)
    xd = x.cuda()
    dev = xd.device
    out = ops.DualLevelResult(y=torch.empty((20, 1024), dtype=torch.bfloat16, device=dev),
                              codes=torch.empty((20, 512), dtype=torch.uint8, device=dev),
                              scales0=torch.empty((20, 2), dtype=torch.float32, device=dev),
                              scales1=torch.empty((20, 32), dtype=torch.uint8, device=dev),
                              mask=torch.empty((20, 128), dtype=torch.uint8, device=dev))
    r = ops.mxfp4_dual_level_qdq(xd, scale_mode="floor", out=out)
    torch.cuda.synchronize()
    assert r is out
    check_all(r, O.dual_level_rowwise(u16(x), 512, 6.0, O.SCALE_FLOOR), "out buffers")
    bad = ops.DualLevelResult(y=None, codes=None, scales0=torch.empty((20, 3), dtype=torch.float32, device=dev),
                              scales1=torch.empty((20, 32), dtype=torch.uint8, device=dev))
    with pytest.raises(ValueError):
        ops.mxfp4_dual_level_qdq(xd, out=bad)
    bad = ops.DualLevelResult(y=None, codes=None, scales0=torch.empty((20, 2), dtype=torch.float64, device=dev),
                              scales1=torch.empty((20, 32), dtype=torch.uint8, device=dev))
    with pytest.raises(TypeError):
        ops.mxfp4_dual_level_qdq(xd, out=bad)
