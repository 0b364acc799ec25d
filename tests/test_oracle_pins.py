"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test derives the expected values a different way from the oracle:
hand-computed golden blocks, an exact squared-mantissa test for round(log2 r),
frexp for floor(log2 amax), a brute-force nearest-code search with an explicit
tie rule, algebraic invariants (power-of-two scaling, sign symmetry,
idempotence, codebook round trip), padding and transposition identities for
the whole-tensor drivers, and numpy's cumsum for group_list normalisation.

Source of the method: amct pull request 264, mxfp4_qat/fake_quant.py
(_block_scale, _round_to_e2m1, _quant_dequant_torch, mxfp4_saturation_mask,
_MXFP4FakeQuantSTE) and the MindSpore fake_w4a8_gmm_func.py page
(normalize_group_list).
"""
from __future__ import annotations

import numpy as np
import pytest

from tests.golden.load import load

CODES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MODES = {"page": 0, "floor": 1}


# --------------------------------------------------------------------------- helpers

def bf16_from_f32(a: np.ndarray) -> np.ndarray:
    """Exact fp32 -> bf16 bits; asserts the value is representable."""
    u = np.asarray(a, np.float32).view(np.uint32)
    assert not np.any(u & 0xFFFF), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def widen(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def all_finite_bf16() -> np.ndarray:
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


def expected_k_page(amax: np.ndarray, sf: float) -> np.ndarray:
    """round(log2(max(fl32(amax/sf), 2^-30))) without log2: r = m * 2^e with
    m in [1, 2); round(log2 r) = e + (m*m >= 2), exact in float64."""
    with np.errstate(over="ignore"):
        r = (amax.astype(np.float32) / np.float32(sf)).astype(np.float32)
    r = np.maximum(r, np.float32(2.0 ** -30))
    f, E = np.frexp(r.astype(np.float64))  # r = f * 2^E, f in [0.5, 1)
    m = f * 2.0
    k = (E - 1) + (m * m >= 2.0)
    return np.where(np.isinf(r), 1000, k)  # fl32(amax/sf) overflowed: log2 = +inf


def expected_k_floor(amax: np.ndarray) -> np.ndarray:
    f, E = np.frexp(amax.astype(np.float64))
    k = (E - 1) - 2
    k = np.where(amax == 0, -127, k)
    return np.maximum(k, -127)


def nearest_code_ties_up(ay: np.ndarray):
    """Brute-force nearest E2M1 magnitude, ties to the larger code."""
    best = np.zeros(ay.shape, np.int64)
    bestd = np.abs(ay - CODES[0])
    for i in range(1, 8):
        d = np.abs(ay - CODES[i])
        take = d <= bestd  # '<=': a tie goes to the later, larger code
        best = np.where(take, i, best)
        bestd = np.where(take, d, bestd)
    return best


# --------------------------------------------------------------------------- golden

@pytest.mark.parametrize("fname", ["ramp_block.txt", "tie_rule_block.txt",
                                   "mode_discriminator_block.txt", "special_blocks.txt"])
def test_golden_blocks(oracle_mod, fname):
    O = oracle_mod
    head, cases = load(fname)
    sf = float(head["scale_factor"])
    for case in cases:
        inp = case["input"]
        v = widen(inp) if head["dtype"] == "bf16" else inp
        for mname, exp in case["modes"].items():
            out, nib, sat, e8 = O.qdq_block(v, sf, MODES[mname])
            if head["dtype"] == "bf16":
                got = np.array([O.f32_to_bf16(float(o)) for o in out], np.uint16)
            else:
                got = out.view(np.uint32).copy()
                got[np.isnan(out)] = 0x7FC00000
            assert np.array_equal(got, exp["out"]), (case["name"], mname, got, exp["out"])
            assert np.array_equal(nib, exp["nibble"]), (case["name"], mname)
            assert np.array_equal(sat.astype(bool), exp["sat"]), (case["name"], mname)
            assert e8 == exp["e8m0"], (case["name"], mname, e8)


# --------------------------------------------------------------------------- scale rule

@pytest.mark.parametrize("sf", [6.0, 1.0, 4.0, 7.5, 0.75])
def test_page_scale_exhaustive_bf16(oracle_mod, sf):
    amax = np.abs(widen(all_finite_bf16()))
    amax = np.unique(amax)
    k = expected_k_page(amax, sf)
    with np.errstate(over="ignore"):
        exp = np.ldexp(1.0, k).astype(np.float32)  # inf once k >= 128
    got = np.array([oracle_mod.scale_page(float(a), sf) for a in amax], np.float32)
    assert np.array_equal(got, exp)


def test_page_scale_fp32_near_sqrt2_boundaries(oracle_mod):
    rng = np.random.default_rng(7)
    # r = amax/6 whose mantissa sits next to sqrt(2): amax = 6 * sqrt2 * 2^j
    # and its fp32 neighbours, plus random fp32 patterns.
    base = (6.0 * np.sqrt(2.0) * np.ldexp(1.0, np.arange(-40, 120))).astype(np.float32)
    u = base.view(np.uint32).astype(np.int64)
    near = np.concatenate([u + d for d in range(-6, 7)]).astype(np.uint32).view(np.float32)
    rnd = rng.integers(0x00800000, 0x7F000000, 20000, dtype=np.uint32).view(np.float32)
    amax = np.concatenate([near, rnd, np.float32([0.0, 1e-45, 1e-40, 3.4e38])])
    k = expected_k_page(amax, 6.0)
    exp = np.ldexp(1.0, k).astype(np.float32)
    got = np.array([oracle_mod.scale_page(float(a), 6.0) for a in amax], np.float32)
    assert np.array_equal(got, exp)


def test_floor_scale(oracle_mod):
    rng = np.random.default_rng(8)
    amax = np.concatenate([
        np.unique(np.abs(widen(all_finite_bf16()))),
        rng.integers(0, 0x7F800000, 20000, dtype=np.uint32).view(np.float32),
    ])
    k = expected_k_floor(amax)
    exp = np.ldexp(1.0, k).astype(np.float32)
    got = np.array([oracle_mod.scale_floor(float(a)) for a in amax], np.float32)
    assert np.array_equal(got, exp)
    assert np.isnan(oracle_mod.scale_floor(float("nan")))
    assert np.isinf(oracle_mod.scale_page(float("inf"), 6.0))


# --------------------------------------------------------------------------- rounding

@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("mexp", [-126, -60, 0, 17, 40, 100])
@pytest.mark.parametrize("mmant", [6.0, 4.5, 1.0, 7.75])
def test_brute_force_every_bf16_element(oracle_mod, mode, mexp, mmant):
    """Every finite bf16 value v with |v| <= M as element 1 of [M, v, 0 ...]."""
    O = oracle_mod
    M = np.float32(mmant * 2.0 ** mexp)
    vals = all_finite_bf16()
    vals = vals[np.abs(widen(vals)) <= M]
    rows = vals.size
    x = np.zeros((rows, 32), np.uint16)
    x[:, 0] = bf16_from_f32(np.array([M]))[0]
    x[:, 1] = vals
    res = O.qdq_rowwise(x, 32, 6.0, MODES[mode])
    Mv = np.array([M])
    k = int((expected_k_page(Mv, 6.0) if mode == "page" else expected_k_floor(Mv))[0])
    xv = widen(vals).astype(np.float64)
    y = xv / 2.0 ** k  # exact in float64
    idx = nearest_code_ties_up(np.abs(y))
    # sign(fl32(x / 2^k)) is 0 exactly when fl32 rounds |y| to zero: |y| <= 2^-150
    neg = (xv < 0) & (np.abs(y) > 2.0 ** -150)
    val = np.where(neg, -1.0, 1.0) * CODES[idx] * 2.0 ** k
    val = np.where(neg & (idx == 0), -0.0, val)
    exp_out = bf16_from_f32(val.astype(np.float32))
    assert np.array_equal(res["y"][:, 1], exp_out)
    nib = O.unpack_nibbles(res["codes"], 32)
    assert np.array_equal(nib[:, 1], (neg.astype(np.uint8) << 3) | idx.astype(np.uint8))
    sat = O.unpack_bits(res["mask"], 32)
    assert np.array_equal(sat[:, 1], np.abs(xv) > 6.0 * 2.0 ** k)
    assert np.all(res["scales"][:, 0] == k + 127)


# --------------------------------------------------------------------------- invariants

def _rand_bf16(rng, shape, sigma=1.0):
    f = (rng.standard_normal(shape) * sigma).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)  # truncation keeps it a bf16 value


def _shift_exp(b: np.ndarray, j: int) -> np.ndarray:
    """Multiply bf16 values by 2^j exactly (all inputs normal, no overflow)."""
    return bf16_from_f32(widen(b) * np.float32(2.0 ** j))


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("j", [-7, 3, 20])
def test_power_of_two_scale_invariance(oracle_mod, mode, j):
    O = oracle_mod
    rng = np.random.default_rng(11)
    x = _rand_bf16(rng, (256, 256))
    x[(x & 0x7F80) == 0] = 0x3F80  # keep every input normal
    a = O.qdq_rowwise(x, 32, 6.0, MODES[mode])
    b = O.qdq_rowwise(_shift_exp(x, j), 32, 6.0, MODES[mode])
    assert np.array_equal(b["codes"], a["codes"])
    assert np.array_equal(b["scales"].astype(int), a["scales"].astype(int) + j)
    assert np.array_equal(widen(b["y"]), widen(a["y"]) * np.float32(2.0 ** j))
    assert np.array_equal(b["mask"], a["mask"])


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_sign_symmetry(oracle_mod, mode):
    O = oracle_mod
    rng = np.random.default_rng(12)
    x = _rand_bf16(rng, (128, 256))
    a = O.qdq_rowwise(x, 32, 6.0, MODES[mode])
    b = O.qdq_rowwise(x ^ np.uint16(0x8000), 32, 6.0, MODES[mode])
    nz = (x & 0x7FFF) != 0
    assert np.array_equal(b["y"][nz], a["y"][nz] ^ np.uint16(0x8000))
    na, nb = O.unpack_nibbles(a["codes"], 256), O.unpack_nibbles(b["codes"], 256)
    assert np.array_equal(nb[nz], na[nz] ^ 8)
    assert np.array_equal(a["scales"], b["scales"]) and np.array_equal(a["mask"], b["mask"])


@pytest.mark.parametrize("dist", ["normal", "heavy", "tiny"])
def test_floor_mode_idempotent(oracle_mod, dist):
    O = oracle_mod
    rng = np.random.default_rng(13)
    if dist == "normal":
        x = _rand_bf16(rng, (256, 256))
    elif dist == "heavy":
        f = (rng.standard_normal((256, 256)) / np.sqrt(rng.chisquare(4, (256, 256)) / 4)).astype(np.float32)
        x = (f.view(np.uint32) >> 16).astype(np.uint16)
    else:
        x = _rand_bf16(rng, (256, 256), sigma=2.0 ** -128)
    q1 = O.qdq_rowwise(x, 32, 6.0, 1)
    q2 = O.qdq_rowwise(q1["y"], 32, 6.0, 1)
    # equal as values; bitwise they differ only where the first pass wrote -0,
    # which the second maps to +0 (sign(-0) = 0 in _quant_dequant_torch)
    assert np.array_equal(widen(q1["y"]), widen(q2["y"]))
    diff = q1["y"] != q2["y"]
    assert np.all(q1["y"][diff] == 0x8000) and np.all(q2["y"][diff] == 0)


def test_page_mode_fixed_point_when_max_is_6_scale(oracle_mod):
    """Page mode is not idempotent in general (4.5 -> 4 -> 3), but a block whose
    output reaches 6*2^k keeps k and so reproduces itself."""
    O = oracle_mod
    rng = np.random.default_rng(14)
    x = _rand_bf16(rng, (512, 256))
    q1 = O.qdq_rowwise(x, 32, 6.0, 0)
    q2 = O.qdq_rowwise(q1["y"], 32, 6.0, 0)
    yb = widen(q1["y"]).reshape(512, 8, 32)
    k = q1["scales"].astype(np.int64) - 127
    hits = np.abs(yb).max(-1) == 6.0 * np.ldexp(1.0, k)
    assert hits.sum() > 100
    same = (yb == widen(q2["y"]).reshape(512, 8, 32)).all(-1)  # values: -0 == +0
    assert np.all(same[hits])
    # and 4.5 -> 4 -> 3 shows it is not idempotent in general
    blk = np.zeros((1, 32), np.uint16)
    blk[0, 0] = bf16_from_f32(np.array([4.5]))[0]
    blk[0, 1] = bf16_from_f32(np.array([3.0]))[0]
    r1 = O.qdq_rowwise(blk, 32, 6.0, 0)["y"]
    r2 = O.qdq_rowwise(r1, 32, 6.0, 0)["y"]
    assert widen(r1)[0, 0] == 4.0 and widen(r2)[0, 0] == 3.0


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_codebook_round_trip(oracle_mod, mode):
    O = oracle_mod
    rng = np.random.default_rng(15)
    rows = 512
    # page mode clamps the raw scale at 2^-30 (_block_scale), so k >= -30 there
    k = rng.integers(-30 if mode == "page" else -126, 100, rows)
    idx = rng.integers(0, 8, (rows, 32))
    idx[:, 0] = 7
    sgn = np.where(rng.random((rows, 32)) < 0.5, -1.0, 1.0)
    sgn[idx == 0] = 1.0
    v = (sgn * CODES[idx] * np.ldexp(1.0, k)[:, None]).astype(np.float32)
    x = bf16_from_f32(v)
    q = O.qdq_rowwise(x, 32, 6.0, MODES[mode])
    assert np.array_equal(q["y"], x)
    assert np.array_equal(q["scales"][:, 0].astype(np.int64), k + 127)


@pytest.mark.parametrize("mode", ["page", "floor"])
def test_mask_and_packing_consistency(oracle_mod, mode):
    """mask <=> |x| > 6*2^k; mask => |out| = 6*2^k; decode(nibble)*2^(e8m0-127) == out."""
    O = oracle_mod
    rng = np.random.default_rng(16)
    x = _rand_bf16(rng, (256, 200))
    x[:, 7] = np.uint16(0x4248)  # 50.0 outlier column
    q = O.qdq_rowwise(x, 32, 6.0, MODES[mode])
    k = q["scales"].astype(np.int64) - 127
    kk = np.repeat(k, 32, axis=1)[:, :200]
    xv = widen(x).astype(np.float64)
    sat = O.unpack_bits(q["mask"], 200)
    assert np.array_equal(sat, np.abs(xv) > 6.0 * np.ldexp(1.0, kk))
    yv = widen(q["y"]).astype(np.float64)
    assert np.all(np.abs(yv[sat]) == 6.0 * np.ldexp(1.0, kk[sat]))
    nib = O.unpack_nibbles(q["codes"], 200).astype(np.int64)
    dec = np.where(nib & 8, -1.0, 1.0) * CODES[nib & 7] * np.ldexp(1.0, kk)
    assert np.array_equal(dec, yv)
    assert np.array_equal(np.signbit(dec), np.signbit(yv))


# --------------------------------------------------------------------------- drivers

@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("block", [32, 128])
def test_rowwise_tail_block_equals_zero_padded_block(oracle_mod, mode, block):
    """_block_view pads the last dim with zeros: the partial tail block must equal
    the full block formed by appending zeros."""
    O = oracle_mod
    rng = np.random.default_rng(17)
    cols = 3 * block + 5
    x = _rand_bf16(rng, (64, cols))
    q = O.qdq_rowwise(x, block, 6.0, MODES[mode])
    nib = O.unpack_nibbles(q["codes"], cols)
    sat = O.unpack_bits(q["mask"], cols)
    for r in range(64):
        v = np.zeros(block, np.float32)
        v[:5] = widen(x[r, 3 * block:])
        out, nb, st, e8 = O.qdq_block(v, 6.0, MODES[mode])
        assert np.array_equal(q["y"][r, 3 * block:], bf16_from_f32(out[:5]))
        assert np.array_equal(nib[r, 3 * block:], nb[:5])
        assert np.array_equal(sat[r, 3 * block:], st[:5].astype(bool))
        assert q["scales"][r, 3] == e8
        assert np.all(out[5:] == 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("block", [32, 128])
def test_colwise_is_rowwise_of_transpose(oracle_mod, dtype, block):
    O = oracle_mod
    rng = np.random.default_rng(18)
    rows, cols = 2 * block + 9, 37
    x = _rand_bf16(rng, (rows, cols))
    if dtype == "f32":
        x = (rng.standard_normal((rows, cols)) * 3).astype(np.float32)
    c = O.qdq_colwise(x, block, 6.0, 0)
    r = O.qdq_rowwise(np.ascontiguousarray(x.T), block, 6.0, 0)
    assert np.array_equal(c["y"].view(np.uint8), np.ascontiguousarray(r["y"].T).view(np.uint8))
    assert np.array_equal(O.unpack_nibbles(c["codes"], cols), O.unpack_nibbles(r["codes"], rows).T)
    assert np.array_equal(O.unpack_bits(c["mask"], cols), O.unpack_bits(r["mask"], rows).T)
    assert np.array_equal(c["scales"], r["scales"].T)


def test_colwise_groups_equal_per_group_slices(oracle_mod):
    O = oracle_mod
    rng = np.random.default_rng(19)
    counts = np.array([0, 45, 32, 0, 1, 70, 0])
    rows, cols = int(counts.sum()), 48
    x = _rand_bf16(rng, (rows, cols))
    ends = O.group_ends(counts, 1, rows)
    assert np.array_equal(ends, np.cumsum(counts))
    full = O.qdq_colwise(x, 32, 6.0, 1, ends=ends)
    start, srow = 0, 0
    for e in ends:
        if e == start:
            continue
        part = O.qdq_colwise(x[start:e], 32, 6.0, 1)
        s = part["scales"].shape[0]
        assert s == -(-(e - start) // 32)
        assert np.array_equal(full["y"][start:e], part["y"])
        assert np.array_equal(full["codes"][start:e], part["codes"])
        assert np.array_equal(full["mask"][start:e], part["mask"])
        assert np.array_equal(full["scales"][srow:srow + s], part["scales"])
        start, srow = e, srow + s
    assert srow == full["scales"].shape[0] == O.colwise_scale_rows(ends, 32)


def test_group_list_normalisation_and_validation(oracle_mod):
    O = oracle_mod
    assert np.array_equal(O.group_ends([3, 0, 5], 1, 8), [3, 3, 8])
    assert np.array_equal(O.group_ends([3, 3, 8], 0, 8), [3, 3, 8])
    assert O.group_ends([3, 2, 8], 0, 8) is None     # decreasing offsets
    assert O.group_ends([3, 3, 7], 0, 8) is None     # does not cover all rows
    assert O.group_ends([3, -1, 6], 1, 8) is None    # negative count
    assert O.group_ends([-1, 8], 0, 8) is None       # negative offset


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ste_bwd_is_masked_fill(oracle_mod, dtype):
    O = oracle_mod
    rng = np.random.default_rng(20)
    rows, cols = 33, 77
    if dtype == "bf16":
        g = rng.integers(0, 65536, (rows, cols), dtype=np.uint32).astype(np.uint16)
    else:
        g = rng.integers(0, 2 ** 32, (rows, cols), dtype=np.uint64).astype(np.uint32).view(np.float32)
    m = rng.integers(0, 256, (rows, (cols + 7) // 8), dtype=np.uint32).astype(np.uint8)
    bits = O.unpack_bits(m, cols)
    got = O.ste_bwd(g, m, True)
    gb = g.view(np.uint16 if dtype == "bf16" else np.uint32)
    exp = np.where(bits, 0, gb)
    assert np.array_equal(got.view(gb.dtype), exp)
    assert np.array_equal(O.ste_bwd(g, m, False).view(gb.dtype), gb)


def test_torch_page_formula_agrees_on_bf16(oracle_mod):
    """Cross-check against torch CPU ops evaluating the page's fp32 steps
    (log2 / round / exp2 / bucketize). For bf16 inputs fp32 log2 followed by
    round() agrees with the exact nearest integer of log2 for every amax (no
    bf16 amax / 6 lies within fp32 rounding of a half-integer power of two),
    so the two readings give the same bytes here."""
    torch = pytest.importorskip("torch")
    O = oracle_mod
    g = torch.Generator().manual_seed(21)
    xb = (torch.randn(512, 256, generator=g) * 3).to(torch.bfloat16)
    xb[:, 5] *= 40
    xf = xb.float().reshape(512, 8, 32)
    amax = xf.abs().amax(-1, keepdim=True)
    scale = torch.exp2(torch.round(torch.log2(torch.clamp(amax / 6.0, min=2.0 ** -30))))
    y = xf / scale
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    codes = torch.tensor(CODES, dtype=torch.float32)
    q = torch.sign(y) * codes[torch.bucketize(y.abs(), mids, right=True)]
    ref = (q * scale).reshape(512, 256).to(torch.bfloat16)
    res = O.qdq_rowwise(xb.view(torch.int16).numpy().view(np.uint16), 32, 6.0, 0)
    assert np.array_equal(res["y"], ref.view(torch.int16).numpy().view(np.uint16))
    # every finite positive bf16 amax: torch's fp32 scale equals the oracle's
    allb = torch.arange(1, 0x7F80, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    t_scale = torch.exp2(torch.round(torch.log2(torch.clamp(allb / 6.0, min=2.0 ** -30))))
    o_scale = np.array([O.scale_page(float(v), 6.0) for v in allb.tolist()], np.float32)
    assert np.array_equal(t_scale.numpy(), o_scale)


def test_mma_scale_layout_hand_offsets(oracle_mod):
    """Offsets worked out by hand from the cuBLAS "1D block scaling factors
    layout" rule (128 x 4 atoms, atom rows in order, entry (r, c) of an atom
    at 16 (r mod 32) + 4 floor(r / 32) + c) for a 130 x 5 scale matrix: two
    atom rows by two atom columns, 2048 bytes."""
    O = oracle_mod
    s = np.zeros((130, 5), np.uint8)
    expect = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (33, 1): 21, (127, 3): 511,
              (0, 4): 512, (127, 4): 512 + 511 - 3, (128, 0): 1024, (129, 4): 1552}
    for n, (rc, _) in enumerate(expect.items()):
        s[rc] = n + 1
    out = O.mma_scale_layout(s)
    assert out.size == 2048
    for n, (rc, off) in enumerate(expect.items()):
        assert out[off] == n + 1, (rc, off)
    assert np.count_nonzero(out) == len(expect)


@pytest.mark.parametrize("shape", [(128, 4), (130, 5), (256, 56), (1, 1), (300, 7), (513, 224)])
def test_mma_scale_layout_by_reshapes(oracle_mod, shape):
    """The same layout derived by tensor reshapes instead of an index formula:
    pad, cut into 128 x 4 tiles taken tile row by tile row, view each tile as
    4 row-quarters x 32 rows x 4 columns and swap the first two axes."""
    R, C = shape
    rng = np.random.default_rng(R * 1000 + C)
    s = rng.integers(1, 256, shape, dtype=np.uint16).astype(np.uint8)
    n_rb, n_cb = -(-R // 128), -(-C // 4)
    padded = np.zeros((128 * n_rb, 4 * n_cb), np.uint8)
    padded[:R, :C] = s
    tiles = padded.reshape(n_rb, 128, n_cb, 4).transpose(0, 2, 1, 3).reshape(-1, 4, 32, 4)
    ref = tiles.transpose(0, 2, 1, 3).reshape(-1)
    assert np.array_equal(oracle_mod.mma_scale_layout(s), ref)


def test_mma_scale_layout_is_a_placement(oracle_mod):
    """Every entry lands on its own byte; the rest (padding) stays 0."""
    O = oracle_mod
    R, C = 300, 7
    idx = np.arange(R * C, dtype=np.int64).reshape(R, C)
    lo, hi = (idx & 0xFF).astype(np.uint8), (idx >> 8).astype(np.uint8)
    a, b = O.mma_scale_layout(lo), O.mma_scale_layout(hi)
    placed = a.astype(np.int64) | (b.astype(np.int64) << 8)
    nz = O.mma_scale_layout(np.ones((R, C), np.uint8)) == 1
    assert nz.sum() == R * C and placed.size == 512 * 3 * 2
    assert np.array_equal(np.sort(placed[nz]), np.arange(R * C))


def test_threaded_oracle_equals_single_calls():
    """The chunked, threaded runner used by the full-size GPU tests returns
    exactly what one oracle call over the whole array returns (ragged row and
    column counts, groups with empty members and tails, both formats)."""
    import oracle as O
    from tests import oracle_par as OP

    rng = np.random.default_rng(5)
    for rows, cols in ((301, 1000), (64, 4104), (7, 37)):
        xb = rng.integers(0, 1 << 16, (rows, cols), dtype=np.uint64).astype(np.uint16)
        xb[:, ::7] &= 0x3FFF  # plenty of finite values next to the random patterns
        ends = np.cumsum([0, rows // 3, 0, rows - rows // 3]).astype(np.int64)[1:]
        for mode in (O.SCALE_PAGE, O.SCALE_FLOOR):
            for block in (32, 128):
                a, b = OP.qdq_rowwise(xb, block, 6.0, mode), O.qdq_rowwise(xb, block, 6.0, mode)
                for k in a:
                    assert np.array_equal(a[k], b[k]), (rows, cols, k)
                a, b = OP.qdq_colwise(xb, block, 6.0, mode, ends), O.qdq_colwise(xb, block, 6.0, mode, ends)
                for k in a:
                    assert np.array_equal(a[k], b[k]), (rows, cols, k)
        a, b = OP.qdq8_rowwise(xb), O.qdq8_rowwise(xb)
        for k in a:
            assert np.array_equal(a[k], b[k])
        a, b = OP.qdq8_colwise(xb, ends), O.qdq8_colwise(xb, ends)
        for k in a:
            assert np.array_equal(a[k], b[k])
        m = O.qdq_rowwise(xb, 32, 6.0, O.SCALE_PAGE)["mask"]
        assert np.array_equal(OP.ste_bwd(xb, m, True), O.ste_bwd(xb, m, True))


def test_colwise_operand_layout_hand_offsets():
    """The column-wise real-quantisation operand layout, against offsets
    worked out by hand: groups [40, 0, 130] over 3 columns pad to K slots
    [0, 128) and [128, 384); nibble of x[r, c] = (3r + c) mod 16, column-wise
    scale byte (s, c) = 10s + c."""
    import oracle as O

    rows, cols = 170, 3
    r = np.arange(rows)[:, None]
    c = np.arange(cols)[None, :]
    nib = ((3 * r + c) % 16).astype(np.uint8)
    codes = np.zeros((rows, 2), np.uint8)
    codes[:, 0] = nib[:, 0] | (nib[:, 1] << 4)
    codes[:, 1] = nib[:, 2]
    scales = (10 * np.arange(7)[:, None] + np.arange(3)[None, :]).astype(np.uint8)
    ends = np.array([40, 40, 170])
    assert O.colwise_operand_k(ends) == 384
    codesT, sc = O.colwise_operand_layout(codes, scales, ends, cols)
    flat = codesT.reshape(-1)
    assert codesT.shape == (3, 192)
    assert flat[0] == 0x30                 # rows 0, 1 of column 0
    assert flat[192 + 19] == 0x63          # rows 38, 39 of column 1
    assert flat[192 + 20] == 0             # padding of group 0 in column 1
    assert flat[2 * 192 + 64] == 0xDA      # rows 40, 41 (group 2's first slots) of column 2
    assert flat[2 * 192 + 64 + 65] == 0    # slot 130 of group 2: padding
    assert sc.size == 512 * 3
    assert sc[529] == 31                   # column 1, scale column 5 = group 2 block 1 = row 3
    assert sc[34] == 127                   # column 2, scale column 2: padding block of group 0
    assert sc[1024] == 60                  # column 0, scale column 8 = group 2 block 4 = row 6
    assert sc[1024 + 32 + 3] == 127        # column 2, scale column 11: padding
    assert sc[0] == 0 and sc[16 + 1] == 11  # column 0 block 0; column 1 block 1
    # k_alloc wider than needed: the rows get longer, the extra slots stay 0
    codesW, scW = O.colwise_operand_layout(codes, scales, ends, cols, k_alloc=512)
    assert codesW.shape == (3, 256) and np.array_equal(codesW[:, :192], codesT) and not codesW[:, 192:].any()
    assert scW.size == 512 * 4
