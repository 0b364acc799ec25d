"""Page-level API over the CUDA library: differentiable MXFP4 fake quantisation
and a quantisation-aware-training Linear.

Mirrors the public surface of amct pull request 264, mxfp4_qat/fake_quant.py
and linear.py (mxfp4_quant_dequant, mxfp4_saturation_mask, mxfp4_fake_quant,
MXFP4FakeQuantizer, MXFP4QATConfig, MXFP4QATLinear, convert_to_mxfp4_qat),
with the backend switch replaced by the one CUDA path and a scale_mode
argument added ("page": 2^round(log2(amax/scale_factor)), "floor":
2^(floor(log2 amax) - 2)). Blocks run along the last dimension.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.nn.functional as F
from torch import nn

from . import ops

BLOCK_SIZE = 32
SCALE_FACTOR = 6.0
MXFP4_E2M1_MAX = 6.0


def _validate(block_size: int, scale_factor: float, scale_mode: str = "page") -> None:
    # fake_quant.py _validate: non-positive block_size / scale_factor are errors
    if block_size <= 0:
        raise ValueError(f"block_size must be positive, got {block_size}")
    if scale_factor <= 0:
        raise ValueError(f"scale_factor must be positive, got {scale_factor}")
    if block_size not in (32, 128):
        raise ValueError(f"block_size must be 32 or 128 on this path, got {block_size}")
    if scale_mode not in ("page", "floor"):
        raise ValueError(f"scale_mode must be 'page' or 'floor', got {scale_mode!r}")


def mxfp4_quant_dequant(x: torch.Tensor, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                        scale_mode: str = "page") -> torch.Tensor:
    """QDQ without autograd; same shape, dtype and device as x."""
    _validate(block_size, scale_factor, scale_mode)
    if x.ndim == 0:
        raise ValueError("x must have at least 1 dimension")
    r = ops.mxfp4_qdq_fwd(x, block=block_size, scale_factor=scale_factor, scale_mode=scale_mode)
    return r.y_row.view(x.shape)


def unpack_mask(packed: torch.Tensor, cols: int) -> torch.Tensor:
    """Bit-packed [rows, ceil(cols/8)] -> bool [rows, cols]."""
    shifts = torch.arange(8, device=packed.device, dtype=torch.uint8)
    bits = (packed.unsqueeze(-1) >> shifts) & 1
    return bits.reshape(packed.shape[0], -1)[:, :cols].bool()


def mxfp4_saturation_mask(x: torch.Tensor, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                          scale_mode: str = "page") -> torch.Tensor:
    """bool mask, True where |x| > 6 * block scale (the clipped elements)."""
    _validate(block_size, scale_factor, scale_mode)
    r = ops.mxfp4_qdq_fwd(x, block=block_size, scale_factor=scale_factor, scale_mode=scale_mode,
                          emit_values=False, emit_mask=True)
    return unpack_mask(r.mask_row, x.shape[-1]).view(x.shape)


class _MXFP4FakeQuantSTE(torch.autograd.Function):
    """Forward: one kernel writes the QDQ values (and, for the clipped STE, the
    bit-packed saturation mask). Backward: one kernel masks the gradient."""

    @staticmethod
    def forward(ctx, x, block_size, scale_factor, clip_grad, scale_mode):
        ctx.clip_grad = clip_grad
        ctx.meta = (block_size, scale_factor, scale_mode)
        r = ops.mxfp4_qdq_fwd(x, block=block_size, scale_factor=scale_factor, scale_mode=scale_mode,
                              emit_mask=clip_grad)
        if clip_grad:
            ctx.save_for_backward(r.mask_row)
        return r.y_row.view(x.shape)

    @staticmethod
    def backward(ctx, grad_output):
        if not ctx.clip_grad:
            return grad_output, None, None, None, None
        (mask,) = ctx.saved_tensors
        block_size, scale_factor, scale_mode = ctx.meta
        g = ops.mxfp4_ste_bwd(grad_output.contiguous(), saved_mask=mask, clip_grad=True, block=block_size,
                              scale_factor=scale_factor, scale_mode=scale_mode)
        return g, None, None, None, None


def mxfp4_fake_quant(x: torch.Tensor, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                     clip_grad: bool = False, scale_mode: str = "page") -> torch.Tensor:
    """Differentiable MXFP4 fake quantisation with a plain or clipped STE."""
    _validate(block_size, scale_factor, scale_mode)
    return _MXFP4FakeQuantSTE.apply(x, block_size, scale_factor, clip_grad, scale_mode)


class MXFP4FakeQuantizer(nn.Module):
    """Stateless module form of mxfp4_fake_quant (no parameters or buffers, so a
    model's state_dict is unchanged by inserting it)."""

    def __init__(self, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                 clip_grad: bool = False, scale_mode: str = "page") -> None:
        super().__init__()
        _validate(block_size, scale_factor, scale_mode)
        self.block_size = block_size
        self.scale_factor = scale_factor
        self.clip_grad = clip_grad
        self.scale_mode = scale_mode

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return mxfp4_fake_quant(x, self.block_size, self.scale_factor, self.clip_grad, self.scale_mode)

    def extra_repr(self) -> str:
        return (f"block_size={self.block_size}, scale_factor={self.scale_factor}, "
                f"clip_grad={self.clip_grad}, scale_mode={self.scale_mode!r}")


@dataclasses.dataclass
class MXFP4QATConfig:
    """Settings shared by converted layers (quantize_input=False is W4A16)."""

    quantize_weight: bool = True
    quantize_input: bool = False
    block_size: int = BLOCK_SIZE
    scale_factor: float = SCALE_FACTOR
    clip_grad: bool = False
    scale_mode: str = "page"

    def __post_init__(self) -> None:
        _validate(self.block_size, self.scale_factor, self.scale_mode)

    def make_quantizer(self) -> MXFP4FakeQuantizer:
        return MXFP4FakeQuantizer(self.block_size, self.scale_factor, self.clip_grad, self.scale_mode)


class MXFP4QATLinear(nn.Linear):
    """nn.Linear computing F.linear(Q(x), Q(W), b); the bias is not quantised and
    the master weight stays in its own precision (the STE routes its gradient)."""

    def __init__(self, in_features: int, out_features: int, bias: bool = True, device=None, dtype=None,
                 config: MXFP4QATConfig | None = None) -> None:
        super().__init__(in_features, out_features, bias, device=device, dtype=dtype)
        self.config = config if config is not None else MXFP4QATConfig()
        self.weight_quantizer = self.config.make_quantizer() if self.config.quantize_weight else None
        self.input_quantizer = self.config.make_quantizer() if self.config.quantize_input else None

    @classmethod
    def from_linear(cls, linear: nn.Linear, config: MXFP4QATConfig | None = None) -> "MXFP4QATLinear":
        """Adopt an existing layer's Parameter objects (no copy, optimiser state stays valid)."""
        layer = cls(linear.in_features, linear.out_features, bias=linear.bias is not None, device="meta",
                    dtype=linear.weight.dtype, config=config)
        layer.weight = linear.weight
        if linear.bias is not None:
            layer.bias = linear.bias
        return layer

    def forward(self, input: torch.Tensor) -> torch.Tensor:
        if self.input_quantizer is not None:
            input = self.input_quantizer(input)
        w = self.weight if self.weight_quantizer is None else self.weight_quantizer(self.weight)
        return F.linear(input, w, self.bias)


def convert_to_mxfp4_qat(module: nn.Module, config: MXFP4QATConfig | None = None,
                         skip_names: tuple[str, ...] = ()) -> nn.Module:
    """Replace every nn.Linear (subclasses included) under module in place;
    dotted paths containing any of skip_names are left alone; converting twice
    is a no-op. Returns module."""

    def walk(m: nn.Module, prefix: str) -> None:
        for name, child in list(m.named_children()):
            path = prefix + name
            if any(s in path for s in skip_names) or isinstance(child, MXFP4QATLinear):
                continue
            if isinstance(child, nn.Linear):
                setattr(m, name, MXFP4QATLinear.from_linear(child, config))
            else:
                walk(child, path + ".")

    walk(module, "")
    return module
