"""CPU proof of the division step of the dual-level kernel.

The dual-level reading (sglang mxfp4_npu.py, NPUMXFP4DiffusionLinearMethod;
level-1 input y = fl32(x / s0)) needs the IEEE fp32 quotient of every element
by its level-0 scale. The kernel forms it from the block's reciprocal with
one fma correction where that is exact, and falls back to the IEEE division
elsewhere. dual_level_division_check.c replays those steps in C for every
pair of a bf16 level-0 amax and a bf16 element of a block it can head, with
both signs, and counts the pairs where the corrected product differs from
x / s0 in any bit; the count must be zero. It also checks the kernel's
table for s0 = fl32(a0 / 6) and fl32(1 / s0): the entries for a0's
significand at exponent 0, shifted by a0's exponent, for every a0 >= 2^-65."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_corrected_reciprocal_product_is_the_ieee_quotient(tmp_path):
    exe = tmp_path / "divcheck"
    base = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
            os.path.join(HERE, "dual_level_division_check.c"), "-lm"]
    if subprocess.run(base[:1] + ["-fopenmp"] + base[1:], capture_output=True).returncode != 0:
        subprocess.run(base, check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True, timeout=600).stdout.split()
    got = dict(zip(out[0::2], map(int, out[1::2])))
    assert got["pairs"] == 2 * sum(range(1, 0x7F80)), got  # every (a0, x) pair with 0 < |x| <= a0
    assert got["fast"] > got["pairs"] // 2, got            # the corrected product covers most pairs
    assert got["bad"] == 0, got
    assert got["table"] == 0x7F80 - (62 << 7) and got["table_bad"] == 0, got
