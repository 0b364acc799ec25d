"""The torch binding's argument handling on the GPU: inputs whose rows the C
ABI cannot address directly (expanded, overlapping), caller-supplied output
buffers that do not fit the call, and invalid group lists, which every entry
point reports instead of returning undefined outputs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from mxfp4_block_fake_b200 import MXFP4ArgumentError, ops, workloads as W

pytestmark = pytest.mark.gpu


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_expanded_and_overlapping_inputs_are_read_as_their_values():
    row = W.mixed(1, 64, seed=3).cuda()
    expanded = row.expand(8, 64)  # row stride 0
    r = ops.mxfp4_qdq_fwd(expanded, rowwise=True, colwise=True, emit_codes=True, emit_mask=True)
    ref = ops.mxfp4_qdq_fwd(expanded.contiguous(), rowwise=True, colwise=True, emit_codes=True, emit_mask=True)
    for k in ("y_row", "y_col", "codes_row", "codes_col", "mask_row", "mask_col", "scales_row"):
        assert torch.equal(getattr(r, k).view(torch.uint8), getattr(ref, k).view(torch.uint8)), k
    store = W.mixed(1, 64 * 8, seed=4).cuda().view(-1)
    overlap = store.as_strided((8, 64), (16, 1))  # rows overlap by 48 elements
    r = ops.mxfp4_qdq_fwd(overlap, emit_codes=True)
    exp = O.qdq_rowwise(u16(overlap), 32, 6.0, O.SCALE_PAGE)
    assert np.array_equal(u16(r.y_row), exp["y"]) and np.array_equal(r.codes_row.cpu().numpy(), exp["codes"])
    g = torch.ones(1, 64, dtype=torch.bfloat16, device="cuda").expand(8, 64)
    gi = ops.mxfp4_ste_bwd(g, x=expanded, clip_grad=True)
    exp_g = O.ste_bwd(u16(g), O.qdq_rowwise(u16(expanded), 32, 6.0, O.SCALE_PAGE)["mask"], True)
    assert np.array_equal(u16(gi), exp_g)


def test_output_buffers_that_do_not_fit_are_rejected():
    x = W.mixed(64, 256, seed=5).cuda()
    r = ops.alloc_outputs(x, block=32, rowwise=True, colwise=True, num_groups=0, emit_codes=True, emit_mask=True)
    wide = torch.empty(64, 512, dtype=x.dtype, device="cuda")
    r.y_col = wide[:, :256]  # a different row pitch than y_row
    with pytest.raises(ValueError):
        ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True, out=r)
    r.y_col = wide[:, :256]
    r.y_row = torch.empty(64, 512, dtype=x.dtype, device="cuda")[:, :256]
    ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True, out=r)  # same pitch on both: accepted
    ref = ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True)
    assert torch.equal(r.y_row.contiguous().view(torch.int16), ref.y_row.view(torch.int16))
    assert torch.equal(r.y_col.contiguous().view(torch.int16), ref.y_col.view(torch.int16))
    for name, bad in (("codes_row", torch.empty(64, 100, dtype=torch.uint8, device="cuda")),
                      ("mask_col", torch.empty(64, 31, dtype=torch.uint8, device="cuda")),
                      ("scales_col", torch.empty(1, 256, dtype=torch.uint8, device="cuda")),
                      ("codes_col", torch.empty(128, 256, dtype=torch.uint8, device="cuda")[:, :128][::2]),
                      ("y_row", torch.empty(64, 256, dtype=torch.float32, device="cuda"))):
        rr = ops.alloc_outputs(x, block=32, rowwise=True, colwise=True, num_groups=0, emit_codes=True,
                               emit_mask=True)
        setattr(rr, name, bad)
        with pytest.raises((ValueError, TypeError)):
            ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True, out=rr)
    g = W.mixed(64, 256, seed=6, specials=False).cuda()
    with pytest.raises(ValueError):
        ops.mxfp4_qdq_fwd_bwd(x, g, grad_in=torch.empty(64, 512, dtype=x.dtype, device="cuda")[:, :256])
    with pytest.raises(ValueError):
        ops.mxfp4_ste_bwd(g, x=x, out=torch.empty(256, 64, dtype=x.dtype, device="cuda").t())
    with pytest.raises(ValueError):
        ops.mxfp4_ste_bwd(g, saved_mask=torch.empty(64, 8, dtype=torch.uint8, device="cuda"))


BAD_LISTS = [([50, 40, 60], 0), ([50, 60, 90], 0), ([50, -10, 60], 1), ([-1, 100], 0), ([30, 30], 1)]


@pytest.mark.parametrize("gl,t", BAD_LISTS)
def test_invalid_group_list_raises_from_every_entry_point(gl, t):
    x = W.mixed(100, 128, seed=13).cuda()
    g = W.mixed(100, 128, seed=14, specials=False).cuda()
    glt = torch.tensor(gl, dtype=torch.int64, device="cuda")
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True, group_list=glt, group_list_type=t)
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_qdq_fwd_bwd(x, g, colwise=True, grad_direction="colwise", group_list=glt, group_list_type=t)
    with pytest.raises(MXFP4ArgumentError):
        ops.mxfp4_ste_bwd(g, x=x, clip_grad=True, direction="colwise", group_list=glt, group_list_type=t)
    # asynchronous form: the status word carries the verdict
    r = ops.mxfp4_qdq_fwd(x, rowwise=False, colwise=True, group_list=glt, group_list_type=t, check=False)
    assert r.status is not None and int(r.status.item()) == 1
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ops.mxfp4_ste_bwd(g, x=x, clip_grad=True, direction="colwise", group_list=glt, group_list_type=t,
                      check=False, status=st)
    assert int(st.item()) == 1
    with pytest.raises(ValueError):
        ops.mxfp4_ste_bwd(g, x=x, clip_grad=True, direction="colwise", group_list=glt, group_list_type=t,
                          check=False)


def test_valid_group_list_reports_ok_without_check():
    x = W.mixed(100, 128, seed=13).cuda()
    glt = torch.tensor([40, 0, 60], dtype=torch.int64, device="cuda")
    r = ops.mxfp4_qdq_fwd(x, rowwise=True, colwise=True, group_list=glt, group_list_type=1, check=False,
                          emit_codes=True)
    assert int(r.status.item()) == 0
    exp = O.qdq_colwise(u16(x), 32, 6.0, O.SCALE_PAGE, ends=np.array([40, 40, 100]))
    assert np.array_equal(u16(r.y_col), exp["y"])
