"""QAT layer plumbing that needs no GPU: conversion of a model, parameter
adoption, state_dict invariance and argument validation (amct pull request
264, mxfp4_qat/linear.py: MXFP4QATLinear, from_linear, convert_to_mxfp4_qat;
mxfp4_qat/README_en.md on state_dict compatibility and skip_names)."""
from __future__ import annotations

import pytest
import torch
from torch import nn

from mxfp4_block_fake_b200 import MXFP4FakeQuantizer, MXFP4QATConfig, MXFP4QATLinear, convert_to_mxfp4_qat


class TaggedLinear(nn.Linear):
    """A framework-style Linear subclass (the converter must take it too)."""


class Block(nn.Module):
    def __init__(self):
        super().__init__()
        self.attn = nn.Linear(16, 16)
        self.mlp = nn.Sequential(TaggedLinear(16, 32), nn.GELU(), nn.Linear(32, 16, bias=False))
        self.norm = nn.LayerNorm(16)


class Model(nn.Module):
    def __init__(self):
        super().__init__()
        self.embed_tokens = nn.Embedding(10, 16)
        self.layers = nn.ModuleList([Block(), Block()])
        self.lm_head = nn.Linear(16, 10)


def linear_paths(m: nn.Module, cls=nn.Linear):
    return sorted(n for n, s in m.named_modules() if isinstance(s, cls))


def test_converts_nested_linears_and_subclasses():
    torch.manual_seed(0)
    m = Model()
    before = linear_paths(m)
    params = {n: p for n, p in m.named_parameters()}
    sd = {k: v.clone() for k, v in m.state_dict().items()}
    out = convert_to_mxfp4_qat(m, MXFP4QATConfig(quantize_input=True))
    assert out is m
    assert linear_paths(m, MXFP4QATLinear) == before  # every Linear, the subclass included
    # the Parameter objects are adopted, not copied
    for n, p in m.named_parameters():
        assert p is params[n], n
    # state_dict: same keys, same tensors
    assert list(m.state_dict().keys()) == list(sd.keys())
    for k, v in m.state_dict().items():
        assert torch.equal(v, sd[k]), k
    q = m.layers[0].mlp[2]
    assert q.bias is None and q.in_features == 32 and q.out_features == 16
    assert isinstance(q.weight_quantizer, MXFP4FakeQuantizer) and isinstance(q.input_quantizer, MXFP4FakeQuantizer)


def test_skip_names_skip_subtrees_and_second_call_is_a_no_op():
    m = Model()
    convert_to_mxfp4_qat(m, skip_names=("lm_head", "layers.1"))
    assert not isinstance(m.lm_head, MXFP4QATLinear)
    assert isinstance(m.layers[0].attn, MXFP4QATLinear)
    assert isinstance(m.layers[0].mlp[0], MXFP4QATLinear)
    assert not any(isinstance(s, MXFP4QATLinear) for s in m.layers[1].modules())
    layers = [s for s in m.modules() if isinstance(s, MXFP4QATLinear)]
    convert_to_mxfp4_qat(m, MXFP4QATConfig(clip_grad=True), skip_names=("lm_head", "layers.1"))
    assert [s for s in m.modules() if isinstance(s, MXFP4QATLinear)] == layers
    assert all(s.config.clip_grad is False for s in layers)


def test_tied_layer_stays_tied_and_root_is_not_replaced():
    shared = nn.Linear(8, 8)
    m = nn.Sequential(shared, nn.ReLU(), shared)
    convert_to_mxfp4_qat(m)
    assert isinstance(m[0], MXFP4QATLinear) and m[0] is m[2]
    assert m[0].weight is shared.weight
    root = nn.Linear(4, 4)
    assert convert_to_mxfp4_qat(root) is root and not isinstance(root, MXFP4QATLinear)


def test_from_linear_keeps_parameters_dtype_and_mode():
    lin = nn.Linear(64, 32).to(torch.bfloat16).eval()
    q = MXFP4QATLinear.from_linear(lin)
    assert q.weight is lin.weight and q.bias is lin.bias
    assert q.weight.dtype == torch.bfloat16 and not q.training and not q.weight_quantizer.training
    assert q.input_quantizer is None  # W4A16 by default
    assert list(dict(q.named_parameters())) == ["weight", "bias"]
    assert "in_features=64, out_features=32" in repr(q)
    # an optimiser built before the conversion still holds the layer's parameters
    opt = torch.optim.SGD(lin.parameters(), lr=0.1)
    assert {id(p) for g in opt.param_groups for p in g["params"]} == {id(q.weight), id(q.bias)}


def test_quantizer_has_no_state_and_describes_itself():
    fq = MXFP4FakeQuantizer(block_size=128, scale_factor=4.0, clip_grad=True, scale_mode="floor")
    assert list(fq.state_dict()) == [] and list(fq.parameters()) == [] and list(fq.buffers()) == []
    assert (fq.block_size, fq.scale_factor, fq.scale_mode, fq.clip_grad) == (128, 4.0, "floor", True)
    assert "128" in repr(fq) and "floor" in repr(fq) and "clipped" in repr(fq)


@pytest.mark.parametrize("kw", [dict(block_size=0), dict(block_size=-32), dict(block_size=64),
                                dict(scale_factor=0.0), dict(scale_factor=-1.0), dict(scale_factor=float("inf")),
                                dict(scale_factor=float("nan")), dict(scale_mode="nearest")])
def test_invalid_settings_are_rejected(kw):
    with pytest.raises(ValueError):
        MXFP4QATConfig(**kw)
    with pytest.raises(ValueError):
        MXFP4FakeQuantizer(**kw)
