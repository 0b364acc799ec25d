"""Quantisation-aware training over the CUDA library.

Public surface (names and signatures as in amct pull request 264,
mxfp4_qat/fake_quant.py and mxfp4_qat/linear.py, so that code written
against that page runs unchanged):

  mxfp4_quant_dequant(x, ...)      fake-quantised copy of x, no autograd
  mxfp4_saturation_mask(x, ...)    bool tensor, True where |x| > 6 * 2^k
  mxfp4_fake_quant(x, ...)         differentiable QDQ, plain or clipped STE
  MXFP4FakeQuantizer               module form of mxfp4_fake_quant
  MXFP4QATConfig                   what a converted layer quantises, and how
  MXFP4QATLinear                   nn.Linear computing linear(Q(x), Q(W), b)
  convert_to_mxfp4_qat(model, ..)  swaps the model's nn.Linear layers in place

Blocks run along the last dimension. Every quantisation is one call of the
library (values and, for the clipped STE, the bit-packed saturation mask in
the same pass); the backward is one masking kernel over the saved mask. The
page's backend switch is not offered: there is one CUDA path. scale_mode
selects the scale rule ("page": 2^round(log2(amax / scale_factor)) with the
2^-30 floor; "floor": 2^max(floor(log2 amax) - 2, -127)).

Nothing here holds a parameter or a buffer of its own: a converted model has
the same state_dict keys and tensors as the float model.
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

_BLOCKS = (32, 128)
_RULES = ("page", "floor")


@dataclasses.dataclass(frozen=True)
class _Spec:
    """One validated quantisation setting (block length, scale divisor, rule)."""

    block: int
    divisor: float
    rule: str

    @staticmethod
    def of(block_size, scale_factor, scale_mode) -> "_Spec":
        if isinstance(block_size, bool) or int(block_size) != block_size or block_size not in _BLOCKS:
            raise ValueError(f"MXFP4 blocks hold 32 or 128 elements here; block_size={block_size!r}")
        sf = float(scale_factor)
        if not sf > 0.0 or sf == float("inf"):
            raise ValueError(f"the scale divisor must be a finite positive number; scale_factor={scale_factor!r}")
        if scale_mode not in _RULES:
            raise ValueError(f"scale_mode selects the scale rule and is 'page' or 'floor'; got {scale_mode!r}")
        return _Spec(int(block_size), sf, scale_mode)

    def qdq(self, x: torch.Tensor, *, values: bool = True, mask: bool = False) -> ops.QDQResult:
        if x.ndim == 0:
            raise ValueError("a 0-dim tensor has no last dimension to block")
        return ops.mxfp4_qdq_fwd(x, block=self.block, scale_factor=self.divisor, scale_mode=self.rule,
                                 emit_values=values, emit_mask=mask)


def unpack_mask(packed: torch.Tensor, cols: int) -> torch.Tensor:
    """Bit-packed saturation mask [rows, ceil(cols/8)] (bit b of byte j is
    column 8j + b) -> bool [rows, cols]."""
    weights = torch.tensor([1 << b for b in range(8)], dtype=torch.uint8, device=packed.device)
    spread = torch.bitwise_and(packed.unsqueeze(-1), weights) != 0
    return spread.flatten(-2)[..., :cols]


def mxfp4_quant_dequant(x: torch.Tensor, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                        scale_mode: str = "page") -> torch.Tensor:
    """x fake-quantised to MXFP4 (same shape, dtype and device); no graph is
    recorded."""
    return _Spec.of(block_size, scale_factor, scale_mode).qdq(x).y_row.view(x.shape)


def mxfp4_saturation_mask(x: torch.Tensor, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                          scale_mode: str = "page") -> torch.Tensor:
    """Where x was clipped: True for |x| > 6 * 2^k of its block (those are the
    elements whose gradient the clipped STE drops)."""
    r = _Spec.of(block_size, scale_factor, scale_mode).qdq(x, values=False, mask=True)
    return unpack_mask(r.mask_row, x.shape[-1]).view(x.shape)


class _MXFP4FakeQuantSTE(torch.autograd.Function):
    """QDQ forward with a straight-through backward. The clipped variant keeps
    the forward's bit-packed saturation mask (one bit per element) and zeroes
    the gradient there; the plain variant passes the gradient unchanged."""

    @staticmethod
    def forward(ctx, x, block_size, scale_factor, clip_grad, scale_mode):
        spec = _Spec.of(block_size, scale_factor, scale_mode)
        r = spec.qdq(x, mask=bool(clip_grad))
        ctx.spec = spec
        ctx.clip = bool(clip_grad)
        if ctx.clip:
            ctx.save_for_backward(r.mask_row)
        return r.y_row.view(x.shape)

    @staticmethod
    def backward(ctx, grad_output):
        g = grad_output
        if ctx.clip:
            (mask,) = ctx.saved_tensors
            s = ctx.spec
            g = ops.mxfp4_ste_bwd(grad_output, saved_mask=mask, clip_grad=True, block=s.block,
                                  scale_factor=s.divisor, scale_mode=s.rule)
        return g, None, None, None, None


def mxfp4_fake_quant(x: torch.Tensor, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                     clip_grad: bool = False, scale_mode: str = "page") -> torch.Tensor:
    """Differentiable MXFP4 fake quantisation: the forward is
    mxfp4_quant_dequant, the backward a straight-through estimator (clip_grad:
    saturated elements get a zero gradient)."""
    _Spec.of(block_size, scale_factor, scale_mode)
    return _MXFP4FakeQuantSTE.apply(x, block_size, scale_factor, clip_grad, scale_mode)


class MXFP4FakeQuantizer(nn.Module):
    """mxfp4_fake_quant as a module. It registers no parameter and no buffer,
    so inserting it leaves a model's state_dict as it was."""

    def __init__(self, block_size: int = BLOCK_SIZE, scale_factor: float = SCALE_FACTOR,
                 clip_grad: bool = False, scale_mode: str = "page") -> None:
        super().__init__()
        self._spec = _Spec.of(block_size, scale_factor, scale_mode)
        self.clip_grad = bool(clip_grad)

    block_size = property(lambda self: self._spec.block)
    scale_factor = property(lambda self: self._spec.divisor)
    scale_mode = property(lambda self: self._spec.rule)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        s = self._spec
        return _MXFP4FakeQuantSTE.apply(x, s.block, s.divisor, self.clip_grad, s.rule)

    def extra_repr(self) -> str:
        s = self._spec
        ste = "clipped" if self.clip_grad else "plain"
        return f"E2M1 x {s.block}, rule={s.rule}, divisor={s.divisor:g}, STE {ste}"


@dataclasses.dataclass
class MXFP4QATConfig:
    """What a converted layer fake-quantises and with which settings. The
    defaults quantise the weight only (W4A16); quantize_input adds the layer
    input (W4A4)."""

    quantize_weight: bool = True
    quantize_input: bool = False
    block_size: int = BLOCK_SIZE
    scale_factor: float = SCALE_FACTOR
    clip_grad: bool = False
    scale_mode: str = "page"

    def __post_init__(self) -> None:
        _Spec.of(self.block_size, self.scale_factor, self.scale_mode)

    def make_quantizer(self) -> MXFP4FakeQuantizer:
        return MXFP4FakeQuantizer(self.block_size, self.scale_factor, self.clip_grad, self.scale_mode)


class MXFP4QATLinear(nn.Linear):
    """nn.Linear whose forward is linear(Q(x), Q(W), b): Q fake-quantises
    (MXFP4, blocks along the input features), the bias stays as it is. The
    optimiser updates the unquantised master weight; the STE carries the
    gradient of Q(W) back to it. As an nn.Linear with stateless quantizers it
    has exactly the float layer's state_dict."""

    def __init__(self, in_features: int, out_features: int, bias: bool = True, device=None, dtype=None,
                 config: MXFP4QATConfig | None = None) -> None:
        super().__init__(in_features, out_features, bias, device=device, dtype=dtype)
        self._attach(config)

    def _attach(self, config: MXFP4QATConfig | None) -> None:
        self.config = MXFP4QATConfig() if config is None else config
        c = self.config
        self.weight_quantizer = c.make_quantizer() if c.quantize_weight else None
        self.input_quantizer = c.make_quantizer() if c.quantize_input else None

    @classmethod
    def from_linear(cls, linear: nn.Linear, config: MXFP4QATConfig | None = None) -> "MXFP4QATLinear":
        """A QAT layer that takes over linear's own Parameter objects: nothing
        is allocated or copied, and an optimiser that already holds those
        parameters keeps training them."""
        layer = cls.__new__(cls)
        nn.Module.__init__(layer)
        layer.in_features, layer.out_features = linear.in_features, linear.out_features
        layer.weight = linear.weight
        layer.register_parameter("bias", linear.bias)
        layer._attach(config)
        layer.train(linear.training)
        return layer

    def forward(self, input: torch.Tensor) -> torch.Tensor:
        w = self.weight if self.weight_quantizer is None else self.weight_quantizer(self.weight)
        x = input if self.input_quantizer is None else self.input_quantizer(input)
        return F.linear(x, w, self.bias)


def convert_to_mxfp4_qat(module: nn.Module, config: MXFP4QATConfig | None = None,
                         skip_names: tuple[str, ...] = ()) -> nn.Module:
    """Swap, in place, every nn.Linear below `module` (subclasses included)
    for an MXFP4QATLinear that adopts its parameters, and return `module`.

    skip_names are substrings of dotted module paths ("encoder.layers.0.fc");
    a module whose path contains one is left as it is, with everything below
    it. Layers that are already MXFP4QATLinear stay untouched, so a second
    call changes nothing. A layer reachable under several paths (tied or
    shared) becomes one QAT layer at all of them. `module` itself is never
    replaced, even when it is an nn.Linear."""
    swaps: list[tuple[str, nn.Linear]] = []
    inside: list[str] = []  # paths of Linear layers: their own children are theirs
    for path, sub in module.named_modules(remove_duplicate=False):
        if not path or any(path.startswith(p + ".") for p in inside):
            continue
        if any(s in path for s in skip_names):
            continue
        if isinstance(sub, nn.Linear):
            inside.append(path)
            if not isinstance(sub, MXFP4QATLinear):
                swaps.append((path, sub))
    made: dict[int, MXFP4QATLinear] = {}
    for path, lin in swaps:
        parent_path, _, name = path.rpartition(".")
        parent = module.get_submodule(parent_path) if parent_path else module
        if id(lin) not in made:
            made[id(lin)] = MXFP4QATLinear.from_linear(lin, config)
        setattr(parent, name, made[id(lin)])
    return module
