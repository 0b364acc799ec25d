"""Pins of the oracle's MXFP8 functions (E4M3 elements, E8M0 scale per 32),
each against a derivation that does not use the oracle: the E4M3 value set
from its bit-field definition, a numpy nearest-even search over every bf16
value, frexp for the scale exponent, torch's own float8_e4m3fn cast, a block
worked by hand, and the transposition identity of the column-wise driver.

Source of the format: [GMM] FakeW4A8GroupedLinear quantises activations and
gradients to MXFP8 (the page names the operators only); the reading follows
the OCP Microscaling rule (scale 2^(floor(log2 amax) - 8), saturated at
2^-127; E4M3 round to nearest even, saturating at 448).
"""
from __future__ import annotations

import numpy as np
import pytest


def e4m3_grid() -> np.ndarray:
    """The 127 finite non-negative E4M3 magnitudes, index = code."""
    c = np.arange(0x7F)
    e, m = (c >> 3) & 15, c & 7
    return np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (e - 7.0))


def nearest_even_codes(y: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of each finite y (ties to the even code, saturation
    above 448, sign bit from y), by brute force over the grid."""
    g = e4m3_grid()
    a = np.abs(y.astype(np.float64))[:, None]
    d = np.abs(a - g[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    even = cand & ((np.arange(0x7F) & 1) == 0)[None, :]
    code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = np.where(np.abs(y) > 448.0, 0x7E, code)
    return (code | np.where(np.signbit(y), 0x80, 0)).astype(np.uint8)


def test_e4m3_value_set(oracle_mod):
    O = oracle_mod
    g = e4m3_grid()
    for c in range(256):
        v = O.e4m3_value(c)
        if c & 0x7F == 0x7F:
            assert np.isnan(v)
            continue
        ref = g[c & 0x7F] * (-1.0 if c & 0x80 else 1.0)
        assert v == ref or (v == 0 and ref == 0), c
        assert O.e4m3_encode(np.float32(ref)) == c, hex(c)
    assert g.max() == 448.0 and g[1] == 2.0 ** -9 and g[8] == 2.0 ** -6


def bf16_values(lo_exp_ok=True) -> np.ndarray:
    b = np.arange(65536, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_e4m3_rounding_every_bf16_value(oracle_mod):
    """Every finite bf16 v below 512 in magnitude, in a block whose maximum
    256 fixes the scale at 2^0: the code is the nearest-even search's."""
    O = oracle_mod
    v = bf16_values()
    v = v[np.abs(v) < 512.0]
    x = np.zeros((v.size, 32), np.float32)
    x[:, 0] = 256.0
    x[:, 1] = v
    r = O.qdq8_rowwise(x)
    assert np.all(r["scales"][:, 0] == 127)
    exp_code = nearest_even_codes(v)
    assert np.array_equal(r["codes"][:, 1], exp_code)
    dec = np.array([O.e4m3_value(int(c)) for c in range(256)])
    assert np.array_equal(r["y"][:, 1], dec[exp_code].astype(np.float32))
    sat = (r["mask"][:, 0] >> 1) & 1
    assert np.array_equal(sat.astype(bool), np.abs(v) > 448.0)


def test_mxfp8_scale_rule_every_bf16_amax(oracle_mod):
    O = oracle_mod
    v = bf16_values()
    v = v[v >= 0]
    x = np.zeros((v.size, 32), np.float32)
    x[:, 3] = v
    r = O.qdq8_rowwise(x)
    m, e = np.frexp(v.astype(np.float64))  # v = m 2^e, m in [0.5, 1): floor(log2 v) = e - 1
    k = np.where(v > 0, np.maximum(e - 1 - 8, -127), -127)
    assert np.array_equal(r["scales"][:, 0].astype(np.int64), k + 127)


def test_e4m3_codes_agree_with_torch_cast(oracle_mod):
    torch = pytest.importorskip("torch")
    O = oracle_mod
    g = torch.Generator().manual_seed(12)
    x = (torch.randn(2048, 64, generator=g) * torch.exp2(torch.randint(-20, 21, (2048, 1), generator=g).float()))
    r = O.qdq8_rowwise(x.numpy())
    xb = x.reshape(2048, 2, 32)
    amax = xb.abs().amax(-1, keepdim=True)
    k = torch.clamp(torch.floor(torch.log2(amax)) - 8, min=-127)
    y = (xb / torch.exp2(k)).reshape(2048, 64)
    ok = y.abs() <= 448
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(r["codes"][ok.numpy()], ref[ok.numpy()])


def test_mxfp8_worked_block(oracle_mod):
    """amax 1.9: floor(log2 1.9) = 0, k = -8 (E8M0 119). 1.0 -> y = 256 = 1.0 *
    2^8, code 0x78, out 1.0; 0.3 -> y = 76.8, nearest E4M3 values 72 and 80,
    80 = 1.25 * 2^6 is nearer: code 0x6A, out 0.3125; -0.3 -> 0xEA, -0.3125;
    1.9 -> y = 486.4 > 448 saturates: code 0x7E, out 1.75, saturated; zeros
    stay +0 with code 0."""
    O = oracle_mod
    x = np.zeros((1, 32), np.float32)
    x[0, :4] = [1.0, 0.3, -0.3, 1.9]
    r = O.qdq8_rowwise(x)
    assert r["scales"][0, 0] == 119
    assert list(r["codes"][0, :5]) == [0x78, 0x6A, 0xEA, 0x7E, 0x00]
    assert list(r["y"][0, :5]) == [1.0, 0.3125, -0.3125, 1.75, 0.0]
    assert r["mask"][0, 0] == 0x08


def test_mxfp8_colwise_is_rowwise_of_transpose(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((96, 40)) * 2.0 ** rng.integers(-30, 30, (96, 1))).astype(np.float32)
    c = O.qdq8_colwise(x)
    r = O.qdq8_rowwise(np.ascontiguousarray(x.T))
    assert np.array_equal(c["y"], r["y"].T)
    assert np.array_equal(c["codes"], r["codes"].T)
    assert np.array_equal(c["scales"], r["scales"].T)


def test_mxfp8_colwise_groups_equal_per_group_slices(oracle_mod):
    """Group restarts: the grouped column-wise result equals the column-wise
    result of each group's rows on their own, scale rows stacked group after
    group; empty groups add no rows."""
    O = oracle_mod
    rng = np.random.default_rng(8)
    counts = [0, 45, 32, 0, 1, 70, 0]
    rows, cols = sum(counts), 24
    x = (rng.standard_normal((rows, cols)) * 2.0 ** rng.integers(-20, 20, (rows, 1))).astype(np.float32)
    ends = np.cumsum(counts)
    g = O.qdq8_colwise(x, ends)
    start, srows = 0, []
    for e in ends:
        if e > start:
            part = O.qdq8_colwise(np.ascontiguousarray(x[start:e]))
            assert np.array_equal(g["y"][start:e], part["y"])
            assert np.array_equal(g["codes"][start:e], part["codes"])
            assert np.array_equal(g["mask"][start:e], part["mask"])
            srows.append(part["scales"])
        start = e
    assert np.array_equal(g["scales"], np.concatenate(srows))


def test_mxfp8_outputs_of_bf16_inputs_are_bf16_values():
    """decode(code) * 2^k is a bf16 value for every bf16 x (|x| below the
    block bound 2^(k+9)), so narrowing it to bf16 is exact; checked at the
    scales where bf16's subnormal range or its top could break it, and
    around 2^0."""
    b = np.arange(65536, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    x = f[np.isfinite(f)].astype(np.float64)
    g = e4m3_grid()
    for k in list(range(-127, -117)) + list(range(-20, 21)) + list(range(110, 120)):
        xs = x[np.abs(x) < 2.0 ** (k + 9)]
        codes = nearest_even_codes((xs * 2.0 ** -k).astype(np.float32))
        out = np.where(codes & 0x80, -1.0, 1.0) * g[codes & 0x7F] * 2.0 ** k
        o32 = out.astype(np.float32)
        assert np.array_equal(o32.astype(np.float64), out), k
        assert np.all((o32.view(np.uint32) & 0xFFFF) == 0), k
