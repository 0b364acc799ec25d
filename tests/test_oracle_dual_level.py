"""Pins of the oracle's dual-level MX quantisation (oracle_dual_level_rowwise)
to facts that do not come from that function.

The sglang page (mxfp4_npu.py, NPUMXFP4DiffusionLinearMethod) names
npu_dynamic_dual_level_mx_quant and its three results (E2M1 codes, a level-0
scale of shape [rows, cols / level0_block], a level-1 scale) and nothing of
their arithmetic, so parity against the page is unpinned. What is pinned here
is the reading the oracle states: s0 = fl32(amax0 / 6) per level-0 block (1
when that is 0), y = fl32(x / s0), the MXFP4 QDQ of amct pull request 264
(mxfp4_qat/fake_quant.py) on y with blocks of 32, out = fl32(code 2^k1 s0)
cast to bf16, and non-finite level-0 blocks written as NaN.

The checks: a hand-worked row (tests/golden/dual_level_block.txt); reduction
to the already pinned single-level QDQ whenever s0 is a power of two; a
brute-force restatement in float64 / numpy float32 with torch's bf16 cast;
power-of-two scale invariance; the special blocks and the ragged tails.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

from tests.golden.load import HERE, _expand

CODES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MODES = {"page": 0, "floor": 1}


def widen(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_bf16_bits(f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits through torch's cast (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(f32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_bf16(shape, seed, scale=1.0) -> np.ndarray:
    g = torch.Generator().manual_seed(seed)
    t = (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


# --------------------------------------------------------------------------- golden row

def load_golden():
    head, modes, mode = {}, {}, None
    with open(os.path.join(HERE, "dual_level_block.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "mode":
                mode = modes.setdefault(vals[0], {})
            elif mode is not None:
                mode[key] = _expand(vals)
            else:
                head[key] = _expand(vals)
    return head, modes


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_golden_row(oracle_mod, mode):
    head, modes = load_golden()
    l0 = int(head["level0_block"][0])
    x = np.array([int(v, 16) for v in head["input"]], np.uint16)[None, :]
    exp = modes[mode]
    r = oracle_mod.dual_level_rowwise(x, l0, float(head["scale_factor"][0]), MODES[mode])
    assert r["scales0"].view(np.uint32).tolist() == [[int(v, 16) for v in head["scales0"]]]
    assert r["y"][0].tolist() == [int(v, 16) for v in exp["out"]]
    nib = oracle_mod.unpack_nibbles(r["codes"], x.shape[1])[0]
    assert nib.tolist() == [int(v) for v in exp["nibble"]]
    sat = np.flatnonzero(oracle_mod.unpack_bits(r["mask"], x.shape[1])[0]).tolist()
    assert sat == [int(v) for v in exp.get("sat", [])]
    assert r["scales1"][0].tolist() == [int(v) for v in exp["scales1"]]


# --------------------------------------------------------------------------- reduction

@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("j", [-3, 0, 5])
def test_power_of_two_level0_scale_reduces_to_single_level(oracle_mod, mode, j):
    """A level-0 block whose amax is 6 * 2^j has s0 = 2^j exactly, so
    y = x * 2^-j without rounding: the outputs, codes and saturation bits
    are the single-level MXFP4 QDQ's, and each E8M0 byte is the single-level
    byte minus j (the blocks stay far from the 2^-30 / 2^-127 scale floors)."""
    rows, cols, l0 = 5, 1536, 512
    x = rand_bf16((rows, cols), 11 + j, 2.0 ** j)
    xf = widen(x).reshape(rows, cols // l0, l0)
    big = np.abs(xf) >= 6 * 2.0 ** j
    xf[big] = np.sign(xf[big]) * 5.5 * 2.0 ** j      # keep |x| < 6 * 2^j
    xf[:, :, 7] = -6 * 2.0 ** j                        # the planted level-0 amax
    xf[0, 1, 64:96] = 0.0                              # one all-zero level-1 block
    x = (xf.reshape(rows, cols).view(np.uint32) >> 16).astype(np.uint16)
    d = oracle_mod.dual_level_rowwise(x, l0, 6.0, MODES[mode])
    s = oracle_mod.qdq_rowwise(x, 32, 6.0, MODES[mode])
    assert np.all(d["scales0"] == np.float32(2.0 ** j))
    assert np.array_equal(d["y"], s["y"])
    assert np.array_equal(d["codes"], s["codes"])
    assert np.array_equal(d["mask"], s["mask"])
    zero_blk = np.zeros_like(s["scales"], bool)
    zero_blk[0, (512 + 64) // 32] = True
    assert np.array_equal(d["scales1"][~zero_blk].astype(int), s["scales"][~zero_blk].astype(int) - j)
    # an all-zero level-1 block sits on the scale floor in both forms
    assert d["scales1"][zero_blk].tolist() == s["scales"][zero_blk].tolist()


# --------------------------------------------------------------------------- brute force

def brute_force(x: np.ndarray, l0: int, sf: float, mode: str):
    """The reading written out without the oracle's loops: numpy float32
    divisions for s0 and y, float64 for everything exact, a nearest-code
    search with ties to the larger code, torch for the bf16 cast."""
    rows, cols = x.shape
    xf = widen(x)
    y_out = np.zeros((rows, cols), np.float32)
    nib = np.zeros((rows, cols), np.uint8)
    sat = np.zeros((rows, cols), bool)
    s0_all = np.zeros((rows, -(-cols // l0)), np.float32)
    s1_all = np.zeros((rows, -(-cols // 32)), np.int64)
    for r in range(rows):
        for j in range(0, cols, l0):
            blk = xf[r, j:j + l0]
            a0 = np.max(np.abs(blk))
            s0 = np.float32(a0) / np.float32(6.0)
            if s0 == 0:
                s0 = np.float32(1.0)
            s0_all[r, j // l0] = s0
            y = (blk / s0).astype(np.float32)
            for b in range(0, blk.size, 32):
                yb = y[b:b + 32].astype(np.float64)
                a1 = np.max(np.abs(yb))
                if mode == "page":
                    raw = max(float(np.float32(a1) / np.float32(sf)), 2.0 ** -30)
                    e = int(np.floor(np.log2(raw)))
                    while 2.0 ** (e + 1) <= raw:
                        e += 1
                    while 2.0 ** e > raw:
                        e -= 1
                    k = e + (1 if raw >= 2.0 ** e * np.sqrt(2.0) else 0)
                else:
                    if a1 == 0:
                        k = -127
                    else:
                        e = int(np.floor(np.log2(a1)))
                        while 2.0 ** (e + 1) <= a1:
                            e += 1
                        while 2.0 ** e > a1:
                            e -= 1
                        k = max(e - 2, -127)
                s1_all[r, (j + b) // 32] = k + 127
                t = np.abs(yb) * 2.0 ** -k
                dist = np.abs(t[:, None] - CODES[None, :])
                best = dist.min(axis=1, keepdims=True)
                idx = np.where(dist == best, np.arange(8), -1).max(axis=1)  # ties: larger code
                q = CODES[idx] * np.where(yb < 0, -1.0, 1.0)
                out = (q * 2.0 ** k * float(s0)).astype(np.float32)
                y_out[r, j + b:j + b + yb.size] = out  # -0 where a negative y rounds to 0
                nib[r, j + b:j + b + yb.size] = np.where(yb < 0, 8, 0) + idx
                sat[r, j + b:j + b + yb.size] = np.abs(yb) > 6.0 * 2.0 ** k
    return to_bf16_bits(y_out), nib, sat, s0_all, s1_all


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("l0,cols,sf", [(64, 200, 6.0), (512, 1100, 6.0), (96, 333, 4.0), (32, 65, 0.75)])
def test_brute_force_restatement(oracle_mod, mode, l0, cols, sf):
    rows = 4
    x = rand_bf16((rows, cols), 3 + cols, 1.0)
    xf = widen(x)
    xf[1, 5] *= 300.0                  # an outlier: most level-1 blocks of that level-0 block go small
    xf[2, : min(64, cols)] *= 2.0 ** -40
    xf[3, :] = np.where(np.arange(cols) % 7 == 0, xf[3, :], 0.0)
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    d = oracle_mod.dual_level_rowwise(x, l0, sf, MODES[mode])
    yb, nib, sat, s0, s1 = brute_force(x, l0, sf, mode)
    assert np.array_equal(d["scales0"], s0)
    assert np.array_equal(d["scales1"].astype(np.int64), s1)
    assert np.array_equal(oracle_mod.unpack_nibbles(d["codes"], cols), nib)
    assert np.array_equal(oracle_mod.unpack_bits(d["mask"], cols), sat)
    assert np.array_equal(d["y"], yb)


# --------------------------------------------------------------------------- invariants and special blocks

@pytest.mark.parametrize("mode", ["page", "floor"])
def test_power_of_two_scale_invariance(oracle_mod, mode):
    """x * 2^m (exact in bf16 here) scales s0 and the outputs by 2^m and
    leaves codes, level-1 bytes and saturation unchanged."""
    x = rand_bf16((3, 1024), 7)
    for m in (-20, 9):
        xm = ((widen(x) * np.float32(2.0 ** m)).view(np.uint32) >> 16).astype(np.uint16)
        a = oracle_mod.dual_level_rowwise(x, 512, 6.0, MODES[mode])
        b = oracle_mod.dual_level_rowwise(xm, 512, 6.0, MODES[mode])
        assert np.array_equal(b["scales0"], a["scales0"] * np.float32(2.0 ** m))
        assert np.array_equal(widen(b["y"]), widen(a["y"]) * np.float32(2.0 ** m))
        for key in ("codes", "scales1", "mask"):
            assert np.array_equal(a[key], b[key])


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_special_level0_blocks(oracle_mod, mode):
    """A NaN or +-inf anywhere in a level-0 block makes the whole block NaN
    (code 0, E8M0 0xFF, no saturation, s0 NaN) and leaves the other level-0
    blocks of the row as they are alone; an all-zero block has s0 = 1."""
    x = rand_bf16((4, 1024 + 100), 9)
    x[0, 3] = 0x7F80      # +inf in block 0 of row 0
    x[1, 600] = 0xFF80    # -inf in block 1 of row 1
    x[2, 1030] = 0x7FC1   # NaN in the ragged block 2 of row 2
    x[3, 512:1024] = 0    # all-zero block 1 of row 3
    d = oracle_mod.dual_level_rowwise(x, 512, 6.0, MODES[mode])
    nib = oracle_mod.unpack_nibbles(d["codes"], x.shape[1])
    bits = oracle_mod.unpack_bits(d["mask"], x.shape[1])
    for r, j in ((0, 0), (1, 1), (2, 2)):
        c0, c1 = 512 * j, min(512 * j + 512, x.shape[1])
        assert np.all(d["y"][r, c0:c1] == 0x7FC0)
        assert np.all(nib[r, c0:c1] == 0) and not bits[r, c0:c1].any()
        assert np.all(d["scales1"][r, c0 // 32:-(-c1 // 32)] == 0xFF)
        assert np.isnan(d["scales0"][r, j]) and d["scales0"][r, j:j + 1].view(np.uint32)[0] == 0x7FC00000
        for jj in range(3):  # the other blocks equal the block quantised on its own
            if jj == j:
                continue
            a0, a1 = 512 * jj, min(512 * jj + 512, x.shape[1])
            alone = oracle_mod.dual_level_rowwise(x[r:r + 1, a0:a1], 512, 6.0, MODES[mode])
            assert np.array_equal(d["y"][r, a0:a1], alone["y"][0])
            assert d["scales0"][r, jj] == alone["scales0"][0, 0]
    assert d["scales0"][3, 1] == 1.0
    assert np.all(d["y"][3, 512:1024] == 0) and np.all(nib[3, 512:1024] == 0)
    assert np.all(d["scales1"][3, 16:32] == (97 if mode == "page" else 0))


def test_level0_block_must_be_a_multiple_of_32(oracle_mod):
    x = rand_bf16((2, 64), 1)
    with pytest.raises(ValueError):
        oracle_mod.dual_level_rowwise(x, 48)
    with pytest.raises(TypeError):
        oracle_mod.dual_level_rowwise(widen(x), 64)
