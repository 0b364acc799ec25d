#!/usr/bin/env python
"""MXFP4 block fake-quant benchmark: effective HBM GB/s of one training step of
the quantiser (QDQ forward + clipped-STE backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of the MoE grouped
activation workload (bf16 [65536, 7168], 256 multinomial groups with empty
ones):
  1. mxfp4_qdq_fwd, both directions from one read of x: row-wise blocks of 32
     and column-wise blocks of 32 restarting at every group offset; writes
     y_row, y_col, packed E2M1 codes and E8M0 scales for both directions and
     the row and column saturation bitmasks;
  2. mxfp4_ste_bwd, clipped STE: grad_in = grad_out with +0 where the saved
     row-wise bitmask is set.
value = algorithmic bytes of all ranks' steps / max-over-ranks device time.
Inputs (x and grad_out, 940 MB each) are larger than the 126 MB L2, so no
flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch
(weak scaling, no data-path collective); NCCL only carries the barrier and
the max-reduction of the timings.

--impl reference times the CPU oracle (tests' reference implementation) on a
bounded sample of the same workload on the host cores; rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MXFP4 QDQ fwd+STE-bwd effective HBM GB/s and % of B200 peak, 1 GPU"
SPEC_PEAK_GBS = 8000.0  # nominal B200 HBM3e figure quoted with the metric
CPU_SAMPLE_ROWS = 16384
REF_SAMPLE_ROWS = 4096


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--scale-mode", choices=["page", "floor"], default="page")
    p.add_argument("--rows", type=int, default=65536)
    p.add_argument("--cols", type=int, default=7168)
    p.add_argument("--groups", type=int, default=256)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-modes", action="store_true",
                   help="skip the extra single-GPU timings of the row-wise and training-step modes")
    p.add_argument("--only-mode", default=None,
                   help="time only this one of the extra modes (its name in the JSON line's modes)")
    return p.parse_args()


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def step_bytes(rows: int, cols: int, s_col: int, esz: int = 2, block: int = 32) -> dict:
    n = rows * cols
    fwd = (n * esz                      # read x
           + 2 * n * esz                # write y_row, y_col
           + 2 * (rows * ((cols + 1) // 2))  # codes row + col
           + rows * ((cols + block - 1) // block) + s_col * cols  # E8M0 scales
           + 2 * rows * ((cols + 7) // 8))   # masks row + col
    bwd = rows * ((cols + 7) // 8) + 2 * n * esz  # read mask + grad_out, write grad_in
    return {"fwd": fwd, "bwd": bwd, "step": fwd + bwd}


def rank_seed(base: int, rank: int) -> int:
    """Every rank quantises its own batch (weak scaling): distinct seeds per rank."""
    return base + 1000 * rank


def reduce_max(values, world: int, device) -> list:
    """Max over ranks of per-rank timings (a no-op for one rank)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_value(bytes_per_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job GB/s: the bytes every rank moved over the slowest rank's time."""
    return bytes_per_step * world * steps / (ms / 1e3) / 1e9


def workload_desc(a, s_col: int) -> dict:
    return {
        "workload": "moe_grouped_dual_qdq_fwd_ste_bwd",
        "shape": [a.rows, a.cols], "dtype": "bf16", "block": 32, "groups": a.groups,
        "group_list": "type 0 cumulative offsets, multinomial sizes p~u^4, 3 forced empty",
        "colwise_scale_rows": s_col, "scale_mode": a.scale_mode,
        "fwd": "row+col QDQ in one pass: y, e2m1 codes, e8m0 scales, saturation bitmasks",
        "bwd": "clipped STE from the saved row-wise bitmask",
        "l2": "inputs larger than L2 (x and grad_out 940 MB each at the default size); no flush",
    }


# ---------------------------------------------------------------------------
# clocks (NVML read-only sampling during the timed region)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_dev: int):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_dev)
            try:
                pci = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(pci)
            except Exception:  # noqa: BLE001 - fall back to the visible index
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_dev)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append(mhz)
                self.reasons |= int(r)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        self._stop = threading.Event()
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": getattr(self, "err", "no samples")}
        reasons = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return 6650.0, "fallback"


def kernel_source_sha() -> str:
    """sha256 over the CUDA sources of the library (the forward kernels)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp4_block_fake_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_for(launch_bytes: int):
    """DRAM traffic per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        sha = kernel_source_sha()
        if t.get("source_sha256") != sha:
            return None
        scale = launch_bytes / t["algorithmic_bytes_per_launch"] if t.get("algorithmic_bytes_per_launch") else 1.0
        return int(t["dram_bytes_per_launch"] * scale)
    except Exception:  # noqa: BLE001
        return None


def run_ours(a, rank: int, world: int):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mxfp4_block_fake_b200 import _abi, ops, workloads as W

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    x_h, counts, offsets = W.moe_grouped(a.rows, a.cols, a.groups, seed=rank_seed(4, rank))
    g_h = W.train_step_grad(a.rows, a.cols, seed=rank_seed(5, rank))
    s_col = ops.mxfp4_colwise_scale_rows(offsets.tolist(), 0, a.rows, 32)
    xd, gd, gl = x_h.cuda(), g_h.cuda(), offsets.cuda()

    res = ops.alloc_outputs(xd, block=32, rowwise=True, colwise=True, num_groups=a.groups, emit_codes=True,
                            emit_mask=True, with_status=True)
    gi = torch.empty_like(gd)
    fargs = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=a.scale_mode,
                          dirs=_abi.ROWWISE | _abi.COLWISE, group_list=gl, group_list_type=0, status=res.status)
    ops._fill_outputs(fargs, res)
    bargs = ops.make_args(gd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.ROWWISE)
    bargs.x = None
    sp = stream.cuda_stream
    mask_ptr, g_ptr, gi_ptr = res.mask_row.data_ptr(), gd.data_ptr(), gi.data_ptr()

    def fwd():
        st = _abi.mxfp4_qdq_fwd(fargs, sp)
        if st:
            _abi.check(st, "mxfp4_qdq_fwd")

    def bwd():
        st = _abi.mxfp4_ste_bwd(bargs, g_ptr, gi_ptr, a.cols, mask_ptr, 1, sp)
        if st:
            _abi.check(st, "mxfp4_ste_bwd")

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[dev])

    for _ in range(a.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    _abi.check(int(res.status.item()), "group_list")
    # soak so the clocks settle before the timed steps
    t0 = time.time()
    while time.time() - t0 < 0.5:
        fwd()
        bwd()
        torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev)
    barrier()
    torch.cuda.synchronize()
    with sampler:
        start.record(stream)
        for i in range(a.steps):
            ev[i][0].record(stream)
            fwd()
            ev[i][1].record(stream)
            bwd()
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms, fwd_ms = reduce_max([start.elapsed_time(end), statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)],
                            world, "cuda")

    # e2e: same step through the public entry points with host buffers. Two
    # device buffer sets, so that the upload of step i+1 runs while the outputs
    # of step i download (PCIe is full duplex); a set's inputs are refilled only
    # after its kernels ran, its outputs rewritten only after they downloaded.
    e2e = None
    if not a.no_e2e:
        xh_p, gh_p = x_h.pin_memory(), g_h.pin_memory()
        sets = []
        for j in range(2):
            xj, gj = (xd, gd) if j == 0 else (torch.empty_like(xd), torch.empty_like(gd))
            rj = res if j == 0 else ops.alloc_outputs(xd, block=32, rowwise=True, colwise=True, num_groups=a.groups,
                                                        emit_codes=True, emit_mask=True, with_status=True)
            gij = gi if j == 0 else torch.empty_like(gi)
            outs = [rj.y_row, rj.y_col, rj.codes_row, rj.scales_row, rj.mask_row, rj.codes_col,
                    rj.scales_col[:s_col], rj.mask_col, gij]
            sets.append((xj, gj, rj, gij, outs))
        outs_h = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in sets[0][4]]
        h2d = xh_p.numel() * 2 + gh_p.numel() * 2
        d2h = sum(o.numel() * o.element_size() for o in sets[0][4])
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        uploaded = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        downloaded = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            j = i & 1
            xj, gj, rj, gij, outs = sets[j]
            up.wait_event(computed[j])
            with torch.cuda.stream(up):
                xj.copy_(xh_p, non_blocking=True)
                gj.copy_(gh_p, non_blocking=True)
            uploaded[j].record(up)
            stream.wait_event(uploaded[j])
            stream.wait_event(downloaded[j])
            ops.mxfp4_qdq_fwd(xj, scale_mode=a.scale_mode, rowwise=True, colwise=True, group_list=gl,
                              emit_codes=True, emit_mask=True, out=rj, check=False)
            ops.mxfp4_ste_bwd(gj, saved_mask=rj.mask_row, clip_grad=True, out=gij)
            computed[j].record(stream)
            down.wait_event(computed[j])
            with torch.cuda.stream(down):
                for o, oh in zip(outs, outs_h):
                    oh.copy_(o, non_blocking=True)
            downloaded[j].record(down)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(a.steps):
            e2e_step(i)
        stream.wait_stream(up)
        stream.wait_stream(down)
        s1.record(stream)
        torch.cuda.synchronize()
        for _, _, rj, _, _ in sets:
            if int(rj.status.item()) != 0:
                raise RuntimeError("e2e: the group_list check failed on the device")
        barrier()
        e2e = (reduce_max([s0.elapsed_time(s1)], world, "cuda")[0], h2d, d2h)

    modes = None
    if world == 1 and not a.no_modes:
        modes = time_modes(a, xd, gd, res, gi, stream, gl, s_col)

    return dict(ms=ms, fwd_ms=fwd_ms, s_col=s_col, clocks=sampler.summary(), e2e=e2e, modes=modes,
                x_h=x_h, g_h=g_h, offsets=offsets, np=np)


def time_modes(a, xd, gd, res, gi, stream, gl, s_col, steps: int = 20):
    """Other modes of the hot path on the same tensors (device-resident, CUDA
    events): row-wise fwd with all outputs + STE from the saved mask, the
    training step of the pages' recipe (row-wise fwd, saved-free STE), and the
    real-quantisation producer (row-wise E2M1 codes + E8M0 scales in the
    block-scaled MMA layout, no dequantised values), blocks of 128 in both
    directions with every output (ungrouped), the MXFP8 element format
    (E4M3, the OCP scale rule) row-wise and in both directions with the
    groups, dual-level MX quantisation (fp32 level-0 scales per 512 elements,
    MXFP4 level 1; every output), and the bench step itself with the other
    scale rule."""
    import torch

    from mxfp4_block_fake_b200 import _abi, ops

    n = a.rows * a.cols
    sp = stream.cuda_stream
    rargs = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.ROWWISE)
    rargs.y_row, rargs.codes_row = res.y_row.data_ptr(), res.codes_row.data_ptr()
    rargs.scales_row, rargs.mask_row = res.scales_row.data_ptr(), res.mask_row.data_ptr()
    rargs.ld_y = a.cols
    vargs = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.ROWWISE)
    vargs.y_row, vargs.ld_y = res.y_row.data_ptr(), a.cols
    bargs = ops.make_args(gd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.ROWWISE)
    bargs.x = None
    rargs_x = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.ROWWISE)
    g_ptr, gi_ptr, m_ptr = gd.data_ptr(), gi.data_ptr(), res.mask_row.data_ptr()
    mma_scales = torch.zeros((ops.scales_row_bytes(a.rows, a.cols, 32, "mma"),), dtype=torch.uint8,
                             device=xd.device)
    margs = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.ROWWISE)
    margs.codes_row, margs.scales_row = res.codes_row.data_ptr(), mma_scales.data_ptr()
    margs.scales_row_layout, margs.ld_y = _abi.SCALES_MMA, a.cols

    def call(st, name):
        if st:
            _abi.check(st, name)

    def row_step():
        call(_abi.mxfp4_qdq_fwd(rargs, sp), "mxfp4_qdq_fwd")
        call(_abi.mxfp4_ste_bwd(bargs, g_ptr, gi_ptr, a.cols, m_ptr, 1, sp), "mxfp4_ste_bwd")

    def train_step():
        call(_abi.mxfp4_qdq_fwd(vargs, sp), "mxfp4_qdq_fwd")
        call(_abi.mxfp4_ste_bwd(rargs_x, g_ptr, gi_ptr, a.cols, None, 1, sp), "mxfp4_ste_bwd")

    def mma_operand():
        call(_abi.mxfp4_qdq_fwd(margs, sp), "mxfp4_qdq_fwd")

    r128 = ops.alloc_outputs(xd, block=128, rowwise=True, colwise=True, num_groups=0, emit_codes=True,
                             emit_mask=True)
    dargs = ops.make_args(xd, block=128, scale_factor=6.0, scale_mode=a.scale_mode,
                          dirs=_abi.ROWWISE | _abi.COLWISE)
    ops._fill_outputs(dargs, r128)

    def dual128():
        call(_abi.mxfp4_qdq_fwd(dargs, sp), "mxfp4_qdq_fwd")

    r8 = ops.alloc_outputs(xd, block=32, rowwise=True, colwise=True, num_groups=a.groups, emit_codes=True,
                           emit_mask=True, with_status=True, elem_format="e4m3")
    row8 = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode="floor", dirs=_abi.ROWWISE, elem_format="e4m3")
    ops._fill_outputs(row8, r8)
    row8.y_col = row8.codes_col = row8.scales_col = row8.mask_col = None
    dual8 = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode="floor", dirs=_abi.ROWWISE | _abi.COLWISE,
                          group_list=gl, group_list_type=0, status=r8.status, elem_format="e4m3")
    ops._fill_outputs(dual8, r8)

    other = "floor" if a.scale_mode == "page" else "page"
    fo_args = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=other, dirs=_abi.ROWWISE | _abi.COLWISE,
                            group_list=gl, group_list_type=0, status=res.status)
    ops._fill_outputs(fo_args, res)
    bo_args = ops.make_args(gd, block=32, scale_factor=6.0, scale_mode=other, dirs=_abi.ROWWISE)
    bo_args.x = None

    def step_other_mode():
        call(_abi.mxfp4_qdq_fwd(fo_args, sp), "mxfp4_qdq_fwd")
        call(_abi.mxfp4_ste_bwd(bo_args, g_ptr, gi_ptr, a.cols, m_ptr, 1, sp), "mxfp4_ste_bwd")

    # the column-wise GEMM operand over the groups (codes + scales, K-major)
    k_op = ops.colwise_operand_k(gl, 0, a.rows)
    opr = ops.alloc_outputs(xd, block=32, rowwise=False, colwise=True, num_groups=a.groups, emit_values=False,
                            emit_codes=True, with_status=True, col_layout="mma", k_alloc=k_op)
    op_args = ops.make_args(xd, block=32, scale_factor=6.0, scale_mode=a.scale_mode, dirs=_abi.COLWISE,
                            group_list=gl, group_list_type=0, status=opr.status)
    ops._fill_outputs(op_args, opr)

    def col_operand():
        call(_abi.mxfp4_qdq_fwd(op_args, sp), "mxfp4_qdq_fwd")

    def mxfp8_row():
        call(_abi.mxfp4_qdq_fwd(row8, sp), "mxfp4_qdq_fwd")

    def mxfp8_dual():
        call(_abi.mxfp4_qdq_fwd(dual8, sp), "mxfp4_qdq_fwd")

    # dual-level MX quantisation (fp32 level-0 scale per 512, MXFP4 level 1), every output
    dl = ops.mxfp4_dual_level_qdq(xd, scale_mode=a.scale_mode, emit_mask=True)
    dl_args = _abi.DualLevelArgs()
    dl_args.x, dl_args.dtype, dl_args.level0_block = xd.data_ptr(), _abi.BF16, 512
    dl_args.rows, dl_args.cols, dl_args.ld, dl_args.ld_y = a.rows, a.cols, a.cols, a.cols
    dl_args.scale_factor, dl_args.scale_mode = 6.0, _abi.SCALE_PAGE if a.scale_mode == "page" else _abi.SCALE_FLOOR
    dl_args.y, dl_args.codes, dl_args.mask = dl.y.data_ptr(), dl.codes.data_ptr(), dl.mask.data_ptr()
    dl_args.scales0, dl_args.scales1 = dl.scales0.data_ptr(), dl.scales1.data_ptr()

    def dual_level():
        call(_abi.mxfp4_dual_level_qdq(dl_args, sp), "mxfp4_dual_level_qdq")

    peak, peak_kind = measured_peaks()
    out = {}
    for name, fn, bpe in (("rowwise_fwd_all_outputs_ste_mask", row_step, 4 + 0.5 + 1 / 32 + 0.125 + 4.125),
                          ("training_step_rowwise_fwd_ste_recompute", train_step, 4 + 6),
                          ("mxfp4_mma_operand_rowwise_codes_scales", mma_operand, 2 + 0.5 + 1 / 32),
                          ("mxfp4_mma_operand_colwise_grouped_codes_scales", col_operand, 2 + 0.5 + 1 / 32),
                          ("dual_block128_all_outputs", dual128, 2 + 4 + 1 + 2 / 128 + 0.25),
                          ("mxfp8_rowwise_all_outputs", mxfp8_row, 2 + 2 + 1 + 1 / 32 + 0.125),
                          ("mxfp8_dual_grouped_all_outputs", mxfp8_dual, 2 + 4 + 2 + 2 / 32 + 0.25),
                          ("dual_level_mx_all_outputs", dual_level, 2 + 2 + 0.5 + 1 / 32 + 4 / 512 + 0.125),
                          (f"bench_step_{other}_scale", step_other_mode, step_bytes(a.rows, a.cols, s_col)["step"] / n)):
        if a.only_mode and name != a.only_mode:
            continue
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        gbs = n * bpe / (ms / 1e3) / 1e9
        out[name] = {"ms_per_step": round(ms, 4), "bytes_per_element": round(bpe, 4), "GB/s": round(gbs, 1),
                     "frac_of_peak": round(gbs / peak, 4), "peak_kind": peak_kind}
    del opr, r8, r128, mma_scales, dl
    torch.cuda.empty_cache()
    if not a.only_mode or a.only_mode.startswith("grouped_gemm"):
        out.update(time_gemm(a, xd, res, gl, stream, steps))
    return out


def bf16_tflops_peak():
    """Dense bf16 tensor-core peak: the measured burst figure, else the
    fallback of this pool (TFLOP/s, kind)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), "measured"
    except Exception:  # noqa: BLE001
        return 1590.0, "fallback"


def time_gemm(a, xd, res, gl, stream, steps: int = 20, n_expert: int = 2048):
    """The grouped block-scaled GEMM that consumes the real-quantisation
    operands: the MoE experts' forward on the bench tokens, D[rows of g] =
    Q(x_g) Q(W_g)^T with one [n_expert, cols] weight per group (seeded
    N(0, 0.02^2) on the device), MXFP4 (kind::mxf4) operands, bf16 output.
    TFLOP/s against the dense bf16 peak times 4 (the nominal FP4 / bf16
    ratio, 9 / 2.25 PFLOP/s)."""
    import torch

    from mxfp4_block_fake_b200 import _abi, ops

    G, K = a.groups, a.cols
    ca, sa = ops.mxfp4_mma_operand(xd)
    sbytes = ops.scales_row_bytes(n_expert, K, 32, "mma")
    wc = torch.empty((G * n_expert, K // 2), dtype=torch.uint8, device=xd.device)
    ws = torch.zeros((G, sbytes), dtype=torch.uint8, device=xd.device)
    gen = torch.Generator(device=xd.device).manual_seed(7)
    for g in range(G):
        w = (torch.randn(n_expert, K, generator=gen, device=xd.device) * 0.02).to(torch.bfloat16)
        ops.mxfp4_qdq_fwd(w, block=32, rowwise=True, emit_values=False, emit_codes=True, scales_layout="mma",
                          out=ops.QDQResult(codes_row=wc[g * n_expert:(g + 1) * n_expert], scales_row=ws[g],
                                            scales_layout="mma"))
    d = torch.empty((a.rows, n_expert), dtype=torch.bfloat16, device=xd.device)
    st = torch.empty((1,), dtype=torch.int32, device=xd.device)
    ga = _abi.GmmArgs()
    ga.elem_format, ga.group_mode = _abi.ELEM_E2M1, _abi.GMM_GROUP_M
    ga.m, ga.n, ga.k = a.rows, n_expert, K
    ga.a, ga.lda, ga.a_scales = ca.data_ptr(), K // 2, sa.data_ptr()
    ga.b, ga.ldb, ga.b_scales = wc.data_ptr(), K // 2, ws.data_ptr()
    ga.group_list, ga.num_groups, ga.group_list_type = gl.data_ptr(), G, 0
    ga.d_dtype, ga.d, ga.ldd, ga.status = _abi.BF16, d.data_ptr(), n_expert, st.data_ptr()
    sp = stream.cuda_stream

    def gemm():
        _abi.check(_abi.mxfp4_grouped_gemm(ga, sp), "mxfp4_grouped_gemm")

    for _ in range(3):
        gemm()
    torch.cuda.synchronize()
    _abi.check(int(st.item()), "mxfp4_grouped_gemm (group_list)")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        gemm()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = 2.0 * a.rows * n_expert * K
    tf = flops / (ms / 1e3) / 1e12
    peak, kind = bf16_tflops_peak()
    return {f"grouped_gemm_mxfp4_moe_fwd_{a.rows}x{n_expert}x{K}_{G}experts": {
        "ms_per_step": round(ms, 4), "TFLOP/s": round(tf, 1), "peak_TFLOP/s": round(4 * peak, 1),
        "peak_kind": f"{kind} bf16 x 4 (nominal fp4/bf16 ratio)", "frac_of_peak": round(tf / (4 * peak), 4)}}


def cpu_baseline(a, x_h, g_h, offsets, rows: int):
    """The oracle, as it stands, on the first `rows` rows of the same batch."""
    import numpy as np
    import torch

    import oracle as O

    rows = min(rows, a.rows)
    xs = x_h[:rows].contiguous().view(torch.int16).numpy().view(np.uint16)
    gs = g_h[:rows].contiguous().view(torch.int16).numpy().view(np.uint16)
    ends = np.minimum(offsets.numpy(), rows)
    ends = ends[: int(np.searchsorted(ends, rows)) + 1]
    ends[-1] = rows
    mode = O.SCALE_PAGE if a.scale_mode == "page" else O.SCALE_FLOOR
    s_col = O.colwise_scale_rows(ends, 32)
    t0 = time.perf_counter()
    r = O.qdq_rowwise(xs, 32, 6.0, mode)
    O.qdq_colwise(xs, 32, 6.0, mode, ends=ends)
    O.ste_bwd(gs, r["mask"], True)
    dt = time.perf_counter() - t0
    b = step_bytes(rows, a.cols, s_col)["step"]
    return dict(value=b / dt / 1e9, seconds=dt, rows=rows, s_col=s_col)


def _oracle_warm(_):
    """Pool warm-up: import the oracle (loads its C library) in the worker."""
    import oracle  # noqa: F401

    return os.getpid()


def _oracle_chunk(job):
    """One worker of the all-cores baseline: the oracle on rows [r0, r1) of
    the batch (whole groups), read from memory-mapped files."""
    import numpy as np

    import oracle as O

    path_x, path_g, shape, r0, r1, ends, mode = job
    xs = np.ascontiguousarray(np.memmap(path_x, np.uint16, "r", shape=shape)[r0:r1])
    gs = np.ascontiguousarray(np.memmap(path_g, np.uint16, "r", shape=shape)[r0:r1])
    t0 = time.perf_counter()
    r = O.qdq_rowwise(xs, 32, 6.0, mode)
    O.qdq_colwise(xs, 32, 6.0, mode, ends=np.asarray(ends, np.int64))
    O.ste_bwd(gs, r["mask"], True)
    return time.perf_counter() - t0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_all_cores(a, x_h, g_h, offsets, max_procs: int = 64):
    """The oracle, as it stands, on the whole batch, the groups split into
    contiguous chunks over one process per host core (spawned; the oracle
    itself is single-threaded). Wall time of the chunks (each reads its rows
    from a memory-mapped copy of the batch), pool warm-up excluded."""
    import multiprocessing as mp
    import shutil
    import tempfile

    import numpy as np
    import torch

    import oracle as O

    procs = max(1, min(os.cpu_count() or 1, max_procs))
    ends = offsets.numpy().astype(np.int64)
    rows = a.rows
    # split at group ends nearest to equal row counts
    cuts = [0]
    for k in range(1, procs):
        target = k * rows // procs
        e = int(ends[int(np.argmin(np.abs(ends - target)))])
        if e > cuts[-1]:
            cuts.append(e)
    if cuts[-1] != rows:
        cuts.append(rows)
    mode = O.SCALE_PAGE if a.scale_mode == "page" else O.SCALE_FLOOR
    xs = x_h.contiguous().view(torch.int16).numpy().view(np.uint16)
    gs = g_h.contiguous().view(torch.int16).numpy().view(np.uint16)
    tmp = tempfile.mkdtemp(prefix="mxfp4_cpu_baseline_")
    try:
        path_x, path_g = os.path.join(tmp, "x.u16"), os.path.join(tmp, "g.u16")
        xs.tofile(path_x)
        gs.tofile(path_g)
        jobs = []
        for r0, r1 in zip(cuts[:-1], cuts[1:]):
            local = ends[(ends > r0) & (ends <= r1)] - r0
            if len(local) == 0 or local[-1] != r1 - r0:
                local = np.append(local, r1 - r0)
            jobs.append((path_x, path_g, xs.shape, r0, r1, local.tolist(), mode))
        ctx = mp.get_context("spawn")
        with ctx.Pool(len(jobs)) as pool:
            pool.map(_oracle_warm, range(len(jobs)))
            t0 = time.perf_counter()
            pool.map(_oracle_chunk, jobs, chunksize=1)
            wall = time.perf_counter() - t0
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    s_col = O.colwise_scale_rows(ends, 32)
    b = step_bytes(rows, a.cols, s_col)["step"]
    return dict(value=b / wall / 1e9, seconds=wall, cores=len(jobs))


def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if a.impl == "reference":
        if rank != 0:
            return
        run_reference(a)
        return

    import torch
    import torch.distributed as dist

    if world > 1:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        r = run_ours(a, rank, world)
        if rank == 0:
            peak, peak_kind = measured_peaks()
            b = step_bytes(a.rows, a.cols, r["s_col"])
            value = weak_value(b["step"], a.steps, world, r["ms"])
            achieved = b["fwd"] / (r["fwd_ms"] / 1e3) / 1e9
            line = {
                "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(r["ms"] / a.steps, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,1) bf16, multinomial groups)",
                "config": workload_desc(a, r["s_col"]),
                "pct_of_peak": {f"{peak_kind}_copy_{int(peak)}": round(100 * value / world / peak, 1),
                                "spec_8000": round(100 * value / world / SPEC_PEAK_GBS, 1)},
                "elements_per_s": round(a.rows * a.cols * world * a.steps / (r["ms"] / 1e3), 1),
                "parts_ms": {"qdq_fwd_dual": round(r["fwd_ms"], 4),
                             "ste_bwd": round(r["ms"] / a.steps - r["fwd_ms"], 4)},
                "roofline": {"bound": "hbm", "kernel": "qdq_staged_kernel (dual, grouped, bf16, block 32)",
                             "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                             "unit": "GB/s", "frac": round(achieved / peak, 4),
                             "traffic": traffic_for(b["fwd"]),
                             "algorithmic_bytes_per_launch": b["fwd"]},
                "gpu_launches": 2 * a.steps,
                "clocks": r["clocks"],
            }
            if r["modes"] is not None:
                line["modes"] = r["modes"]
            if r["e2e"] is not None:
                ms_e, h2d, d2h = r["e2e"]
                line["e2e"] = {"value": round(weak_value(b["step"], a.steps, world, ms_e), 2),
                               "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                               "ms_per_step": round(ms_e / a.steps, 3)}
            if world == 1 and not a.no_cpu_baseline:
                cb = cpu_baseline(a, r["x_h"], r["g_h"], r["offsets"], CPU_SAMPLE_ROWS)
                line["cpu_baseline"] = {
                    "value": round(cb["value"], 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                    "sample": f"first {cb['rows']} of {a.rows} rows x {a.cols} cols of the same batch "
                              f"(groups cut at the sample end), one full step, {cb['seconds']:.1f} s"}
                try:
                    cp = cpu_baseline_all_cores(a, r["x_h"], r["g_h"], r["offsets"])
                    line["cpu_baseline_all_cores"] = {
                        "value": round(cp["value"], 4), "unit": "GB/s", "cores": cp["cores"], "kind": "oracle",
                        "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                        "sample": f"the whole batch ({a.rows} x {a.cols}), one full step, groups split into "
                                  f"{cp['cores']} contiguous chunks, one spawned process each, "
                                  f"{cp['seconds']:.1f} s wall"}
                except Exception as e:  # noqa: BLE001 - a baseline, not the measurement
                    line["cpu_baseline_all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


def run_reference(a):
    import numpy as np

    from mxfp4_block_fake_b200 import workloads as W

    x_h, counts, offsets = W.moe_grouped(a.rows, a.cols, a.groups, seed=4)
    g_h = W.train_step_grad(a.rows, a.cols, seed=5)
    for _ in range(a.warmup):
        cpu_baseline(a, x_h, g_h, offsets, REF_SAMPLE_ROWS)
    tot_b, tot_s = 0, 0.0
    for _ in range(a.steps):
        cb = cpu_baseline(a, x_h, g_h, offsets, REF_SAMPLE_ROWS)
        tot_b += step_bytes(cb["rows"], a.cols, cb["s_col"])["step"]
        tot_s += cb["seconds"]
    value = tot_b / tot_s / 1e9
    s_col = int(np.sum((np.diff(np.concatenate([[0], offsets.numpy()])) + 31) // 32))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * tot_s / a.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, multinomial groups)", "config": workload_desc(a, s_col),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: first {REF_SAMPLE_ROWS} rows x {a.cols} cols of the batch"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
