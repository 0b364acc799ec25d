"""mxfp4_block_fake_b200: MXFP4 block fake quantisation (QDQ + clipped STE) on
NVIDIA B200, behind the C ABI of include/mxfp4.h (libmxfp4.so).

Layers:
  libmxfp4.so         sm_100a kernels + C ABI (csrc/mxfp4.cu)
  _abi                ctypes mirror of the C ABI
  ops                 the entry points over torch CUDA tensors
  qat                 autograd STE function, quantizer module, QAT Linear
  workloads           seeded synthetic inputs
"""
from ._abi import MXFP4ArgumentError, MXFP4Error
from .ops import (
    DualLevelResult,
    QDQResult,
    colwise_scale_rows_bound,
    mxfp4_colwise_scale_rows,
    mxfp4_dual_level_qdq,
    mxfp4_qdq_fwd,
    mxfp4_qdq_fwd_bwd,
    mxfp4_ste_bwd,
)
from .qat import (
    MXFP4FakeQuantizer,
    MXFP4QATConfig,
    MXFP4QATLinear,
    convert_to_mxfp4_qat,
    mxfp4_fake_quant,
    mxfp4_quant_dequant,
    mxfp4_saturation_mask,
    unpack_mask,
)

__all__ = [
    "MXFP4Error", "MXFP4ArgumentError", "QDQResult", "DualLevelResult", "mxfp4_dual_level_qdq", "colwise_scale_rows_bound", "mxfp4_colwise_scale_rows",
    "mxfp4_qdq_fwd", "mxfp4_qdq_fwd_bwd", "mxfp4_ste_bwd", "MXFP4FakeQuantizer", "MXFP4QATConfig",
    "MXFP4QATLinear", "convert_to_mxfp4_qat", "mxfp4_fake_quant", "mxfp4_quant_dequant",
    "mxfp4_saturation_mask", "unpack_mask",
]
