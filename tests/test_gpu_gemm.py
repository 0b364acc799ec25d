"""GPU checks of the grouped block-scaled GEMM (tcgen05 tensor cores) against
the oracle: the operands are this library's real-quantisation outputs, the
reference is the float64 product of the oracle's fake-quantised matrices
(MindSpore hyper-parallel fake_w4a8_gmm_func.py, FakeW4A8GroupedLinear.
grouped_matmul: "NN"/"NT" group the rows of the left operand, "TN" the
contraction over each group's tokens).

Every product of two dequantised values is exact in fp32 (E2M1 x E2M1 has
at most 4 significant bits, E4M3 x E4M3 at most 8, times powers of two), so
the fp32 accumulation differs from the exact sum only by the rounding of the
partial sums: |D - ref| <= K 2^-24 sum_k |a_k b_k| (+ the bf16 output
rounding, 2^-8 |ref|, when D is bf16).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import MXFP4ArgumentError, ops

pytestmark = pytest.mark.gpu


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def deq(y16: np.ndarray) -> np.ndarray:
    return O.bf16_to_f32(y16).astype(np.float64)


def rand_bf16(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16)


def check(d: torch.Tensor, ref: np.ndarray, mag: np.ndarray, k: int, bf16_out: bool):
    got = d.float().cpu().numpy().astype(np.float64)
    bound = k * 2.0 ** -24 * mag + (2.0 ** -8 * np.abs(ref) if bf16_out else 0.0) + 1e-300
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), f"max err/bound {float((err / bound).max()):.3f}"


def mxfp8_rowwise(x: torch.Tensor):
    r = ops.mxfp4_qdq_fwd(x, block=32, scale_mode="floor", rowwise=True, emit_values=False, emit_codes=True,
                          scales_layout="mma", elem_format="e4m3")
    return r.codes_row, r.scales_row


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("counts", [[300], [128, 0, 77, 200, 1], [0, 513, 0]])
def test_grouped_over_rows(fmt, out_dtype, counts):
    """'NN'/'NT': tokens x [M, K] in groups, one weight W_g [N, K] per group,
    D[rows of g] = Q(x_g) Q(W_g)^T."""
    M, N, K = sum(counts), 192, 512
    G = len(counts)
    x = rand_bf16(M, K, 1)
    ws = [rand_bf16(N, K, 10 + g, 0.05) for g in range(G)]
    xd = x.cuda()
    if fmt == "e2m1":
        ca, sa = ops.mxfp4_mma_operand(xd)
        parts = [ops.mxfp4_mma_operand(w.cuda()) for w in ws]
        qx = deq(O.qdq_rowwise(u16(x), 32, 6.0, O.SCALE_PAGE)["y"])
        qw = [deq(O.qdq_rowwise(u16(w), 32, 6.0, O.SCALE_PAGE)["y"]) for w in ws]
    else:
        ca, sa = mxfp8_rowwise(xd)
        parts = [mxfp8_rowwise(w.cuda()) for w in ws]
        qx = deq(O.qdq8_rowwise(u16(x))["y"])
        qw = [deq(O.qdq8_rowwise(u16(w))["y"]) for w in ws]
    cb = torch.cat([p[0].view(torch.uint8) for p in parts])
    sb = torch.cat([p[1].view(torch.uint8) for p in parts])
    gl = torch.tensor(counts, dtype=torch.int64, device="cuda")
    d = ops.mxfp4_grouped_gemm(ca, sa, cb, sb, gl, k=K, group_mode="m", elem_format=fmt, group_list_type=1,
                               out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = np.zeros((M, N))
    mag = np.zeros((M, N))
    r0 = 0
    for g, n in enumerate(counts):
        ref[r0:r0 + n] = qx[r0:r0 + n] @ qw[g].T
        mag[r0:r0 + n] = np.abs(qx[r0:r0 + n]) @ np.abs(qw[g]).T
        r0 += n
    check(d, ref, mag, K, out_dtype == torch.bfloat16)


@pytest.mark.parametrize("mode", ["page", "floor"])
@pytest.mark.parametrize("counts", [[200, 0, 77, 328, 5], [1000], [0, 0, 129]])
def test_grouped_over_k_weight_gradient(mode, counts):
    """'TN': per group, dW_g = Qc(x_g)^T Qc(dy_g) with the column-wise
    (group-restarting) operands in the K-major operand layout; an empty
    group's product is zero."""
    T = sum(counts)
    cx, cy = 256, 320
    x = rand_bf16(T, cx, 2)
    dy = rand_bf16(T, cy, 3, 1e-3)
    ends = np.cumsum(counts)
    a, sa, ka = ops.mxfp4_colwise_mma_operand(x.cuda(), group_list=counts, group_list_type=1, scale_mode=mode)
    b, sb, kb = ops.mxfp4_colwise_mma_operand(dy.cuda(), group_list=counts, group_list_type=1, scale_mode=mode)
    assert ka == kb
    gl = torch.tensor(counts, dtype=torch.int64, device="cuda")
    d = ops.mxfp4_grouped_gemm(a, sa, b, sb, gl, k=ka, group_mode="k", elem_format="e2m1", group_list_type=1,
                               k_rows=T, out_dtype=torch.float32)
    torch.cuda.synchronize()
    mm = O.SCALE_PAGE if mode == "page" else O.SCALE_FLOOR
    qx = deq(O.qdq_colwise(u16(x), 32, 6.0, mm, ends=ends)["y"])
    qy = deq(O.qdq_colwise(u16(dy), 32, 6.0, mm, ends=ends)["y"])
    r0 = 0
    for g, n in enumerate(counts):
        ref = qx[r0:r0 + n].T @ qy[r0:r0 + n]
        mag = np.abs(qx[r0:r0 + n]).T @ np.abs(qy[r0:r0 + n])
        check(d[g], ref, mag, max(n, 1), False)
        r0 += n


def test_invalid_group_lists_are_reported():
    K, N = 256, 128
    x = rand_bf16(200, K, 4).cuda()
    ca, sa = ops.mxfp4_mma_operand(x)
    cb, sb = ops.mxfp4_mma_operand(rand_bf16(N, K, 5).cuda())
    with pytest.raises(MXFP4ArgumentError):  # does not add up to the rows
        ops.mxfp4_grouped_gemm(ca, sa, cb, sb, torch.tensor([150], dtype=torch.int64, device="cuda"), k=K,
                               group_list_type=1)
    with pytest.raises(ValueError):  # k not a multiple of 128
        ops.mxfp4_grouped_gemm(ca, sa, cb, sb, [200], k=200, group_list_type=1)
    a, s_a, ka = ops.mxfp4_colwise_mma_operand(x, group_list=[200], group_list_type=1)
    with pytest.raises(MXFP4ArgumentError):  # groups need more K slots than k_alloc
        ops.mxfp4_grouped_gemm(a, s_a, a, s_a, torch.tensor([1, 1, 198], dtype=torch.int64, device="cuda"),
                               k=ka, group_mode="k", group_list_type=1, k_rows=200)


@pytest.mark.parametrize("mode", ["m", "k"])
def test_many_tiles_per_cta(mode):
    """Enough output tiles that every CTA of the persistent grid takes
    several in turn (the stage ring and both accumulators wrap many times),
    against the oracle on every output."""
    if mode == "m":
        counts = [5000, 0, 3000, 8384]
        M, N, K = sum(counts), 1024, 512
        x = rand_bf16(M, K, 21)
        ws = [rand_bf16(N, K, 30 + g, 0.05) for g in range(len(counts))]
        ca, sa = ops.mxfp4_mma_operand(x.cuda())
        parts = [ops.mxfp4_mma_operand(w.cuda()) for w in ws]
        cb = torch.cat([p[0].view(torch.uint8) for p in parts])
        sb = torch.cat([p[1].view(torch.uint8) for p in parts])
        gl = torch.tensor(counts, dtype=torch.int64, device="cuda")
        d = ops.mxfp4_grouped_gemm(ca, sa, cb, sb, gl, k=K, group_list_type=1)
        qx = deq(O.qdq_rowwise(u16(x), 32, 6.0, O.SCALE_PAGE)["y"])
        r0 = 0
        for g, n in enumerate(counts):
            qw = deq(O.qdq_rowwise(u16(ws[g]), 32, 6.0, O.SCALE_PAGE)["y"])
            ref = qx[r0:r0 + n] @ qw.T
            mag = np.abs(qx[r0:r0 + n]) @ np.abs(qw).T
            check(d[r0:r0 + n], ref, mag, K, False)
            r0 += n
    else:
        counts = [300, 450, 0, 250]
        T, cx, cy = sum(counts), 2048, 1536
        x = rand_bf16(T, cx, 22)
        dy = rand_bf16(T, cy, 23, 1e-3)
        a, sa, ka = ops.mxfp4_colwise_mma_operand(x.cuda(), group_list=counts, group_list_type=1)
        b, sb, _ = ops.mxfp4_colwise_mma_operand(dy.cuda(), group_list=counts, group_list_type=1)
        gl = torch.tensor(counts, dtype=torch.int64, device="cuda")
        d = ops.mxfp4_grouped_gemm(a, sa, b, sb, gl, k=ka, group_mode="k", group_list_type=1, k_rows=T)
        ends = np.cumsum(counts)
        qx = deq(O.qdq_colwise(u16(x), 32, 6.0, O.SCALE_PAGE, ends=ends)["y"])
        qy = deq(O.qdq_colwise(u16(dy), 32, 6.0, O.SCALE_PAGE, ends=ends)["y"])
        r0 = 0
        for g, n in enumerate(counts):
            ref = qx[r0:r0 + n].T @ qy[r0:r0 + n]
            mag = np.abs(qx[r0:r0 + n]).T @ np.abs(qy[r0:r0 + n])
            check(d[g], ref, mag, max(n, 1), False)
            r0 += n
