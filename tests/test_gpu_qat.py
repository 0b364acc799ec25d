"""QAT layer on the GPU against the oracle, at 0 ULP.

The tiny QAT linear (fp32 x [4, 64] and W [32, 64] ~ N(0,1), blocks of 32
along the last dimension, y = Q(x) Q(W)^T, grad_out = ones): Q(x), Q(W) and
both saturation masks byte for byte, and y, dx, dW exactly. The sums are
exact: every product of two fake-quantised values has at most four
significant bits and the 64 terms of a dot product span far fewer than 24
bits of exponent, so fp32 accumulation in any order (TF32 included: the
operands have two significant bits) gives the exact value, which float64
also gives. amct pull request 264, mxfp4_qat/linear.py (MXFP4QATLinear) and
fake_quant.py (_MXFP4FakeQuantSTE, mxfp4_saturation_mask).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import (MXFP4FakeQuantizer, MXFP4QATConfig, MXFP4QATLinear, convert_to_mxfp4_qat,
                                   mxfp4_fake_quant, mxfp4_quant_dequant, mxfp4_saturation_mask)
from mxfp4_block_fake_b200 import workloads as W

pytestmark = pytest.mark.gpu

MODES = {"page": O.SCALE_PAGE, "floor": O.SCALE_FLOOR}


def f32_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().contiguous().numpy().view(np.uint32)


def ora_in(x: torch.Tensor) -> np.ndarray:
    x = x.detach().cpu().contiguous()
    return x.view(torch.int16).numpy().view(np.uint16) if x.dtype == torch.bfloat16 else x.numpy()


def ora_bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def exact_f32(a: np.ndarray) -> np.ndarray:
    f = a.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), a), "expected value not representable in fp32"
    return f


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("clip", [False, True])
def test_tiny_qat_linear_exact(mode, clip):
    x, w = W.qat_linear_tiny()
    cfg = MXFP4QATConfig(quantize_input=True, clip_grad=clip, scale_mode=mode)
    lin = MXFP4QATLinear(64, 32, bias=False, config=cfg)
    with torch.no_grad():
        lin.weight.copy_(w)
    lin = lin.cuda()
    xd = x.cuda().requires_grad_(True)
    qx_o = O.qdq_rowwise(x.numpy(), 32, 6.0, MODES[mode])
    qw_o = O.qdq_rowwise(w.numpy(), 32, 6.0, MODES[mode])
    # the operands and the masks, byte for byte
    assert np.array_equal(f32_bits(lin.input_quantizer(xd)), qx_o["y"].view(np.uint32))
    assert np.array_equal(f32_bits(lin.weight_quantizer(lin.weight)), qw_o["y"].view(np.uint32))
    assert np.array_equal(mxfp4_saturation_mask(xd, scale_mode=mode).cpu().numpy(), O.unpack_bits(qx_o["mask"], 64))
    assert np.array_equal(mxfp4_saturation_mask(lin.weight, scale_mode=mode).cpu().numpy(),
                          O.unpack_bits(qw_o["mask"], 64))
    # forward and both gradients, exactly
    y = lin(xd)
    y.backward(torch.ones_like(y))
    qx, qw = qx_o["y"].astype(np.float64), qw_o["y"].astype(np.float64)
    ones = np.ones((4, 32))
    dx, dw = ones @ qw, ones.T @ qx
    if clip:
        dx = np.where(O.unpack_bits(qx_o["mask"], 64), 0.0, dx)
        dw = np.where(O.unpack_bits(qw_o["mask"], 64), 0.0, dw)
    assert np.array_equal(f32_bits(y), exact_f32(qx @ qw.T).view(np.uint32))
    assert np.array_equal(f32_bits(xd.grad), exact_f32(dx).view(np.uint32))
    assert np.array_equal(f32_bits(lin.weight.grad), exact_f32(dw).view(np.uint32))
    if clip:
        # the clipped positions exist in this workload and got +0.0
        assert O.unpack_bits(qw_o["mask"], 64).any()


def test_pull_request_smoke_scenario():
    """The pull request's own check: convert Sequential(Linear(64, 32)) with
    input quantisation, run a batch, back-propagate, finite gradients."""
    torch.manual_seed(0)
    model = torch.nn.Sequential(torch.nn.Linear(64, 32)).cuda()
    convert_to_mxfp4_qat(model, MXFP4QATConfig(quantize_input=True))
    assert isinstance(model[0], MXFP4QATLinear)
    model(torch.randn(4, 64, device="cuda")).sum().backward()
    assert torch.isfinite(model[0].weight.grad).all()
    assert torch.isfinite(model[0].bias.grad).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("mode", ["page", "floor"])
def test_functional_api_on_3d_inputs(dtype, mode):
    """mxfp4_quant_dequant and mxfp4_saturation_mask on a 3-D tensor block its
    last dimension (including a partial tail block) like the oracle on the
    flattened rows; mxfp4_fake_quant's clipped STE on it, with a
    non-contiguous incoming gradient, equals the oracle's STE."""
    x = W.mixed(6 * 5, 100, dtype=dtype, seed=33).view(6, 5, 100)
    xd = x.cuda()
    ora = O.qdq_rowwise(ora_in(x.view(-1, 100)), 32, 6.0, MODES[mode])
    q = mxfp4_quant_dequant(xd, scale_mode=mode)
    assert q.shape == x.shape and q.dtype == dtype
    got = ora_in(q.view(-1, 100))
    assert np.array_equal(got.view(np.uint32) if dtype == torch.float32 else got, ora_bits(ora["y"]))
    m = mxfp4_saturation_mask(xd, scale_mode=mode)
    assert m.shape == x.shape and m.dtype == torch.bool
    assert np.array_equal(m.view(-1, 100).cpu().numpy(), O.unpack_bits(ora["mask"], 100))
    g = W.mixed(100, 6 * 5, dtype=dtype, seed=34, specials=False).cuda().t().reshape(6, 5, 100)
    g = g.transpose(0, 1).contiguous().transpose(0, 1)  # non-contiguous incoming gradient
    assert not g.is_contiguous()
    xr = xd.clone().requires_grad_(True)
    y = mxfp4_fake_quant(xr, clip_grad=True, scale_mode=mode)
    y.backward(g)
    exp = O.ste_bwd(ora_in(g.reshape(-1, 100)), ora["mask"], True)
    got = ora_in(xr.grad.reshape(-1, 100))
    assert np.array_equal(got.view(np.uint32) if dtype == torch.float32 else got, ora_bits(exp))
    # the plain STE passes the gradient through unchanged
    xr.grad = None
    mxfp4_fake_quant(xr, clip_grad=False, scale_mode=mode).backward(g)
    assert torch.equal(xr.grad, g)


def test_quantizer_module_block128_on_bf16_weights():
    w = W.weight_dual(256, 512)
    fq = MXFP4FakeQuantizer(block_size=128, clip_grad=True, scale_mode="floor")
    wd = w.cuda().requires_grad_(True)
    out = fq(wd)
    ora = O.qdq_rowwise(ora_in(w), 128, 6.0, O.SCALE_FLOOR)
    assert np.array_equal(ora_in(out), ora["y"])
    out.backward(torch.ones_like(out))
    exp = np.where(O.unpack_bits(ora["mask"], 512), 0.0, 1.0)
    assert np.array_equal(wd.grad.float().cpu().numpy(), exp)
