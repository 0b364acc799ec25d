"""CPU checks of the C ABI boundary (no GPU needed).

* libmxfp4.so builds, loads and exports every function include/mxfp4.h declares;
* the ctypes mirror of mxfp4_qdq_args has the C layout (sizeof/offsetof taken
  from a C program compiled against the header);
* host-only entry points (scale-row counting, status strings) agree with the
  oracle's group_list normalisation (the MindSpore fake_w4a8_gmm_func.py page,
  normalize_group_list);
* argument errors are rejected on the host before any CUDA call.
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

import numpy as np
import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "mxfp4.h")


@pytest.fixture(scope="module")
def abi():
    from mxfp4_block_fake_b200 import build
    build.build()
    from mxfp4_block_fake_b200 import _abi
    _abi.lib()
    return _abi


def declared_functions() -> list[str]:
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mxfp4_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports(abi):
    assert declared_functions() == sorted(abi.EXPORTS)


def test_library_exports_every_declared_symbol(abi):
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(abi.lib(), name)


@pytest.mark.parametrize("cname,pyname", [("mxfp4_qdq_args", "QdqArgs"), ("mxfp4_gmm_args", "GmmArgs"),
                                          ("mxfp4_dual_level_args", "DualLevelArgs")])
def test_struct_layout_matches_c(abi, tmp_path, cname, pyname):
    cls = getattr(abi, pyname)
    fields = [f for f, _ in cls._fields_]
    src = tmp_path / "layout.c"
    body = "\n".join(f'  printf("{f} %zu\\n", offsetof({cname}, {f}));' for f in fields)
    src.write_text(
        "#include <stdio.h>\n#include <stddef.h>\n#include \"mxfp4.h\"\n"
        "int main(void) {\n" + body + f'\n  printf("sizeof %zu\\n", sizeof({cname}));\n  return 0;\n}}\n'
    )
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), "-o", str(exe), str(src)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                      check=True).stdout.splitlines())
    import ctypes
    for f in fields:
        assert int(got[f]) == getattr(cls, f).offset, f
    assert int(got["sizeof"]) == ctypes.sizeof(cls)


def _gmm(abi, **kw):
    g = abi.GmmArgs()
    g.elem_format, g.group_mode, g.m, g.n, g.k = abi.ELEM_E2M1, abi.GMM_GROUP_M, 256, 128, 256
    g.a, g.lda, g.a_scales = 4096, 128, 8192
    g.b, g.ldb, g.b_scales = 16384, 128, 32768
    g.group_list, g.num_groups, g.group_list_type = 65536, 1, 0
    g.d_dtype, g.d, g.ldd = abi.F32, 131072, 128
    for k, v in kw.items():
        setattr(g, k, v)
    return g


@pytest.mark.parametrize("kw,expected", [
    (dict(elem_format=7), 1), (dict(group_mode=2), 1), (dict(d_dtype=5), 1), (dict(k=200), 1), (dict(k=-128), 1),
    (dict(m=-1), 1), (dict(m=2 ** 31), 2), (dict(group_list=None), 1), (dict(num_groups=0), 1),
    (dict(num_groups=5000), 2), (dict(group_list_type=3), 1), (dict(group_list=65540), 1),
    (dict(group_mode=1, k_rows=-1), 1), (dict(a=None), 1), (dict(lda=64), 1), (dict(lda=136), 1),
    (dict(a=4100), 1), (dict(ldb=100), 1), (dict(d=131076), 1), (dict(ldd=100), 1), (dict(ldd=130), 1),
    (dict(a_scales=8194), 1),
])
def test_grouped_gemm_rejects_bad_arguments_on_host(abi, kw, expected):
    assert abi.mxfp4_grouped_gemm(_gmm(abi, **kw), None) == expected
    assert abi.lib().mxfp4_grouped_gemm(None, None) == abi.EINVAL


def test_header_compiles_as_c_and_cpp(tmp_path):
    src = tmp_path / "inc.c"
    src.write_text('#include "mxfp4.h"\nint f(void) { return MXFP4_ABI_VERSION + MXFP4_MAX_GROUPS; }\n')
    for comp, std in (("gcc", "-std=c99"), ("g++", "-std=c++11")):
        subprocess.run([comp, std, "-Wall", "-Werror", "-c", "-I", os.path.dirname(HEADER), "-x",
                        "c" if comp == "gcc" else "c++", str(src), "-o", str(tmp_path / "o.o")], check=True)


def test_status_strings(abi):
    assert abi.status_string(abi.OK) == "ok"
    assert abi.status_string(abi.EINVAL) == "invalid argument"
    assert abi.status_string(abi.EUNSUPPORTED) == "unsupported argument"
    assert abi.status_string(abi.ECUDA) == "CUDA error"
    assert abi.status_string(77) == "unknown status"
    assert abi.lib().mxfp4_abi_version() == abi.ABI_VERSION


@pytest.mark.parametrize("block", [32, 128])
def test_colwise_scale_rows_matches_oracle(abi, oracle_mod, block):
    rng = np.random.default_rng(3)
    for trial in range(200):
        g = int(rng.integers(1, 40))
        counts = rng.integers(0, 300, g)
        counts[rng.random(g) < 0.3] = 0
        rows = int(counts.sum())
        ends = oracle_mod.group_ends(counts, 1, rows)
        exp = oracle_mod.colwise_scale_rows(ends, block)
        assert abi.mxfp4_colwise_scale_rows(counts.tolist(), 1, rows, block) == exp
        assert abi.mxfp4_colwise_scale_rows(ends.tolist(), 0, rows, block) == exp
        assert abi.mxfp4_colwise_scale_rows_bound(rows, g, block) >= exp
    # invalid lists
    assert abi.mxfp4_colwise_scale_rows([3, 2, 8], 0, 8, 32) == -1
    assert abi.mxfp4_colwise_scale_rows([3, 3, 7], 0, 8, 32) == -1
    assert abi.mxfp4_colwise_scale_rows([3, -1, 6], 1, 8, 32) == -1
    assert abi.mxfp4_colwise_scale_rows(None, 0, 100, 32) == 4


def test_colwise_operand_k_matches_oracle(abi, oracle_mod):
    rng = np.random.default_rng(4)
    L = abi.lib()
    for trial in range(200):
        g = int(rng.integers(1, 40))
        counts = rng.integers(0, 400, g)
        counts[rng.random(g) < 0.3] = 0
        rows = int(counts.sum())
        ends = np.cumsum(counts)
        exp = oracle_mod.colwise_operand_k(ends)
        assert abi.mxfp4_colwise_operand_k(counts.tolist(), 1, rows) == exp
        assert abi.mxfp4_colwise_operand_k(ends.tolist(), 0, rows) == exp
        assert L.mxfp4_colwise_operand_k_bound(rows, g) >= exp
    assert abi.mxfp4_colwise_operand_k(None, 0, 300) == 384
    assert abi.mxfp4_colwise_operand_k([3, 2, 8], 0, 8) == -1
    assert abi.mxfp4_colwise_operand_k([3, -1, 6], 1, 8) == -1
    assert L.mxfp4_colwise_operand_k_bound(300, 0) == 384 and L.mxfp4_colwise_operand_k_bound(-1, 2) == -1
    for cols, k in ((3, 384), (256, 128), (130, 1024), (0, 128)):
        exp = oracle_mod.mma_scale_layout(np.zeros((cols, k // 32), np.uint8)).size if cols else 0
        assert L.mxfp4_colwise_operand_scale_bytes(cols, k) == exp
    assert L.mxfp4_colwise_operand_scale_bytes(10, 100) == -1


def _args(abi, **kw):
    a = abi.QdqArgs()
    a.dtype, a.block, a.rows, a.cols, a.ld = abi.BF16, 32, 4, 64, 64
    a.scale_factor, a.scale_mode, a.dirs = 6.0, abi.SCALE_PAGE, abi.ROWWISE
    a.x = 4096  # never dereferenced: every case below fails host validation first
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,expected", [
    (dict(block=0), 1), (dict(block=-32), 1), (dict(block=64), 2), (dict(block=16), 2),
    (dict(scale_factor=0.0), 1), (dict(scale_factor=-6.0), 1), (dict(scale_factor=float("nan")), 1),
    (dict(scale_factor=float("inf")), 1), (dict(dtype=7), 1), (dict(scale_mode=5), 1),
    (dict(dirs=0), 1), (dict(dirs=4), 1), (dict(rows=-1), 1), (dict(cols=-3), 1),
    (dict(rows=2 ** 31), 2), (dict(x=None), 1), (dict(ld=32), 1), (dict(x=4097), 1),
    (dict(dirs=2, group_list=4096, num_groups=0), 1),
    (dict(dirs=2, group_list=4096, num_groups=5000), 2),
    (dict(dirs=2, group_list=4096, num_groups=3, group_list_type=2), 1),
    (dict(dirs=2, group_list=4097, num_groups=3), 1),
    (dict(scales_row_layout=2), 1), (dict(elem_format=2), 1), (dict(elem_format=-1), 1),
    (dict(elem_format=1), 2),                               # MXFP8 in PAGE mode
    (dict(elem_format=1, scale_mode=1, block=128), 2),      # MXFP8 with blocks of 128
    (dict(col_layout=2), 1), (dict(col_layout=-1), 1),
    # column-wise GEMM operand layout: k_alloc, dtype and alignment are checked on the host
    (dict(dirs=2, codes_col=8192, col_layout=1, k_alloc=100), 1),
    (dict(dirs=2, codes_col=8192, col_layout=1, k_alloc=0), 1),
    (dict(dirs=2, codes_col=8192, col_layout=1, k_alloc=128, rows=200), 1),
    (dict(dirs=2, codes_col=8200, col_layout=1, k_alloc=128), 1),
    (dict(dirs=2, scales_col=8193, col_layout=1, k_alloc=128), 1),
    (dict(dirs=2, codes_col=8192, col_layout=1, k_alloc=128, dtype=0), 2),
    (dict(dirs=2, codes_col=8192, col_layout=1, k_alloc=128, block=128), 2),
    (dict(dirs=2, codes_col=8192, col_layout=1, k_alloc=128, scale_factor=100.0), 2),
    (dict(dirs=3, codes_col=8192, col_layout=1, k_alloc=100, y_row=8192), 1),
])
def test_fwd_rejects_bad_arguments_on_host(abi, kw, expected):
    assert abi.mxfp4_qdq_fwd(_args(abi, **kw), None) == expected


@pytest.mark.parametrize("rows,cols,block", [(130, 160, 32), (128, 128, 32), (1, 1, 32), (300, 7168, 32),
                                             (257, 1000, 128), (0, 64, 32)])
def test_scales_row_bytes(abi, oracle_mod, rows, cols, block):
    L = abi.lib()
    nblk = -(-cols // block)
    assert L.mxfp4_scales_row_bytes(rows, cols, block, abi.SCALES_ROWMAJOR) == rows * nblk
    mma = oracle_mod.mma_scale_layout(np.zeros((rows, nblk), np.uint8)).size if rows else 0
    assert L.mxfp4_scales_row_bytes(rows, cols, block, abi.SCALES_MMA) == mma
    assert L.mxfp4_scales_row_bytes(rows, cols, block, 7) == -1
    assert L.mxfp4_scales_row_bytes(-1, cols, block, abi.SCALES_ROWMAJOR) == -1


def _dual(abi, **kw):
    a = abi.DualLevelArgs()
    a.x, a.dtype, a.level0_block, a.rows, a.cols, a.ld = 4096, abi.BF16, 512, 4, 1024, 1024
    a.scale_factor, a.scale_mode, a.ld_y = 6.0, abi.SCALE_PAGE, 1024
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,expected", [
    (dict(rows=-1), 1), (dict(cols=-2), 1), (dict(dtype=3), 1), (dict(level0_block=0), 1),
    (dict(level0_block=48), 1), (dict(level0_block=-512), 1), (dict(scale_factor=0.0), 1),
    (dict(scale_factor=float("nan")), 1), (dict(scale_factor=float("inf")), 1), (dict(scale_mode=2), 1),
    (dict(dtype=0), 2), (dict(level0_block=256), 2), (dict(level0_block=1024), 2),
    (dict(x=None), 1), (dict(ld=1000), 1), (dict(y=8192, ld_y=1000), 1),
    (dict(rows=0), 0), (dict(cols=0, x=None), 0), (dict(rows=2 ** 30), 2), (dict(cols=2 ** 30, ld=2 ** 30), 2),
])
def test_dual_level_rejects_bad_arguments_on_host(abi, kw, expected):
    assert abi.mxfp4_dual_level_qdq(_dual(abi, **kw), None) == expected
    assert abi.lib().mxfp4_dual_level_qdq(None, None) == abi.EINVAL


def test_null_args_and_bad_bwd_arguments(abi):
    import ctypes
    L = abi.lib()
    assert L.mxfp4_qdq_fwd(None, None) == abi.EINVAL
    assert L.mxfp4_ste_bwd(None, 4096, 4096, 64, None, 1, None) == abi.EINVAL
    a = _args(abi, dirs=3)
    assert abi.mxfp4_ste_bwd(a, 4096, 4096, 64, None, 1, None) == abi.EINVAL  # two directions
    a = _args(abi)
    assert abi.mxfp4_ste_bwd(a, None, 4096, 64, None, 1, None) == abi.EINVAL
    assert abi.mxfp4_ste_bwd(a, 4096, 4096, 32, None, 1, None) == abi.EINVAL  # ld_grad < cols
    assert abi.mxfp4_qdq_fwd_bwd(a, 4096, None, 64, 1, None) == abi.EINVAL
    assert abi.mxfp4_qdq_fwd_bwd(a, 4096, 4096, 64, 2, None) == abi.EINVAL  # grad dir not computed
    assert abi.mxfp4_qdq_fwd_bwd(a, 4096, 4096, 64, 3, None) == abi.EINVAL
    _ = ctypes


def test_product_path_has_no_cpu_fallback():
    torch = pytest.importorskip("torch")
    from mxfp4_block_fake_b200 import mxfp4_quant_dequant
    with pytest.raises(ValueError, match="CUDA"):
        mxfp4_quant_dequant(torch.ones(4, 64))
    from mxfp4_block_fake_b200 import mxfp4_dual_level_qdq
    with pytest.raises(ValueError, match="CUDA"):
        mxfp4_dual_level_qdq(torch.ones(4, 512, dtype=torch.bfloat16))


def test_product_code_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "mxfp4_block_fake_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "liboracle" not in text and "mxfp4_oracle" not in text, f
    _ = sys


def test_layout_predicate_copies_expanded_and_overlapping_inputs():
    """The binding passes a tensor's own pitch to the library only when its
    rows are [rows][ld] with ld >= cols and unit column stride; expanded
    (row stride 0), overlapping (0 < row stride < cols) and transposed
    inputs are copied first."""
    import torch

    from mxfp4_block_fake_b200.ops import rows_addressable

    base = torch.zeros(8, 64)
    assert rows_addressable(tuple(base.shape), tuple(base.stride()))
    padded = torch.zeros(8, 80)[:, :64]
    assert rows_addressable(tuple(padded.shape), tuple(padded.stride()))
    expanded = torch.zeros(1, 64).expand(8, 64)
    assert expanded.stride(0) == 0
    assert not rows_addressable(tuple(expanded.shape), tuple(expanded.stride()))
    overlap = torch.zeros(200).as_strided((8, 64), (16, 1))
    assert not rows_addressable(tuple(overlap.shape), tuple(overlap.stride()))
    transposed = torch.zeros(64, 8).t()
    assert not rows_addressable(tuple(transposed.shape), tuple(transposed.stride()))
    one_row = torch.zeros(1, 64).expand(1, 64)
    assert rows_addressable(tuple(one_row.shape), tuple(one_row.stride()))
    one_col = torch.zeros(8, 5)[:, 2:3]
    assert rows_addressable(tuple(one_col.shape), tuple(one_col.stride()))
