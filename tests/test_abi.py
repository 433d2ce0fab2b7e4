"""The C-ABI library without a GPU: it loads, exports every entry point the header
declares, and its host-side checks return the documented status before any launch."""
import ctypes
import os
import re

import pytest

import combine_moe_dispatch_04_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe_dc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 9
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(moe.EXPORTS)


def _call_layout(shape, **kw):
    args = dict(idx=ctypes.c_void_p(16), mask=None, counts=ctypes.c_void_p(16),
                send=ctypes.c_void_p(16), assist=ctypes.c_void_p(16), status=None,
                ws=ctypes.c_void_p(256), ws_bytes=1 << 30)
    args.update(kw)
    return moe.moe_dispatch_layout(ctypes.byref(shape.c()), args["idx"], args["mask"],
                                   args["counts"], args["send"], args["assist"], args["status"],
                                   args["ws"], args["ws_bytes"], None)


GOOD = moe.Shape(bs=4096, k=8, h=1536, num_experts=64)


@pytest.mark.parametrize("field,value,status", [
    ("k", 0, moe.MOE_ERR_ARG), ("k", 17, moe.MOE_ERR_ARG), ("num_experts", 0, moe.MOE_ERR_ARG),
    ("num_experts", 1025, moe.MOE_ERR_ARG), ("bs", -1, moe.MOE_ERR_ARG),
    ("h", 1028, moe.MOE_ERR_ALIGN), ("dtype", 7, moe.MOE_ERR_ARG),
    ("mask_ndim", 3, moe.MOE_ERR_ARG), ("zero_expert_num", -1, moe.MOE_ERR_ARG),
    ("a_capacity", 4096 * 8 - 1, moe.MOE_ERR_CAPACITY),
])
def test_shape_checks(field, value, status):
    import dataclasses
    bad = dataclasses.replace(GOOD, **{field: value})
    assert _call_layout(bad) == status


def test_capacity_follows_min_of_experts_and_k():
    # [combine] Constraints at one device: A >= BS * min(E, K); with E = 4 < K = 8
    # (4 zero experts make K <= N) the bound is BS * 4. Only invalid calls are
    # made here: no GPU is needed.
    sh = dict(bs=100, k=8, h=1024, num_experts=4, zero_expert_num=4)
    assert _call_layout(moe.Shape(**sh, a_capacity=399)) == moe.MOE_ERR_CAPACITY
    assert _call_layout(moe.Shape(**sh, a_capacity=400),
                        idx=None) == moe.MOE_ERR_ARG  # capacity accepted, null idx caught


def test_k_larger_than_id_range():
    assert _call_layout(moe.Shape(bs=8, k=5, h=1024, num_experts=4)) == moe.MOE_ERR_ARG
    assert _call_layout(moe.Shape(bs=8, k=5, h=1024, num_experts=4, zero_expert_num=1),
                        idx=None) == moe.MOE_ERR_ARG  # K <= N accepted, null idx caught


# Above 16384 tokens the layout runs in tiles and needs a workspace.
TILED = moe.Shape(bs=20000, k=8, h=1536, num_experts=64)


def test_null_pointers_and_workspace():
    assert _call_layout(GOOD, idx=None) == moe.MOE_ERR_ARG
    assert _call_layout(GOOD, assist=None) == moe.MOE_ERR_ARG
    assert _call_layout(TILED, ws=None) == moe.MOE_ERR_CAPACITY
    need = moe.moe_layout_workspace_bytes(ctypes.byref(TILED.c()))
    t = (20000 + 255) // 256
    assert need == 4 * (t * 64 + 64 + t)  # tile counts, expert totals, tile status words
    assert _call_layout(TILED, ws_bytes=need - 1) == moe.MOE_ERR_CAPACITY
    assert _call_layout(TILED, ws=ctypes.c_void_p(8)) == moe.MOE_ERR_ALIGN
    masked = moe.Shape(bs=64, k=8, h=1536, num_experts=64, mask_ndim=2)
    assert _call_layout(masked) == moe.MOE_ERR_ARG  # mask_ndim 2 without a mask


def test_other_entry_points_check_first():
    s = ctypes.byref(GOOD.c())
    p = ctypes.c_void_p(256)
    # quant mode outside {0, 2}
    assert moe.moe_dispatch_permute(s, p, p, None, 1, p, p, None) == moe.MOE_ERR_ARG
    # quant mode 2 needs dynamic_scales
    assert moe.moe_dispatch_permute(s, p, p, None, 2, p, None, None) == moe.MOE_ERR_ARG
    # misaligned row pointer
    assert moe.moe_dispatch_permute(s, ctypes.c_void_p(258), p, None, 0, p, None, None) == \
        moe.MOE_ERR_ALIGN
    # smooth-scaled int8 dispatch: every pointer required, smooth scales 16-byte aligned,
    # H a multiple of 16 and at most 16384
    sm = moe.moe_dispatch_permute_smooth
    assert sm(s, p, p, p, p, None, p, p, None) == moe.MOE_ERR_ARG
    assert sm(s, p, None, p, p, p, p, p, None) == moe.MOE_ERR_ARG
    assert sm(s, p, p, p, p, ctypes.c_void_p(260), p, p, None) == moe.MOE_ERR_ALIGN
    h8 = moe.Shape(bs=16, k=2, h=1032, num_experts=4)
    assert sm(ctypes.byref(h8.c()), p, p, p, p, p, p, p, None) == moe.MOE_ERR_ALIGN
    big = moe.Shape(bs=16, k=2, h=16400, num_experts=4)
    assert sm(ctypes.byref(big.c()), p, p, p, p, p, p, p, None) == moe.MOE_ERR_UNSUPPORTED
    # copy/const experts need ori_x; const experts need alpha_1, alpha_2, v
    sp = moe.Shape(bs=16, k=4, h=1024, num_experts=8, copy_expert_num=1, const_expert_num=1)
    args = [p, p, p, p, None, None, None, None, p, p, p, p, None]
    assert moe.moe_combine_fwd(ctypes.byref(sp.c()), *args) == moe.MOE_ERR_ARG
    args[7] = p  # ori_x
    args[8] = None  # alpha_1 missing
    assert moe.moe_combine_fwd(ctypes.byref(sp.c()), *args) == moe.MOE_ERR_ARG
    # combine comm_quant_mode outside {0, 2}
    args2 = [p, p, p, p, None, None, None, None, None, None, None]
    assert moe.moe_combine_fwd_comm_quant(s, *args2, 1, p, None) == moe.MOE_ERR_ARG
    # the workspace variant: 16-byte aligned, large enough, and ep_send_counts with it
    ws = moe.moe_combine_fwd_comm_quant_workspace_bytes(s)
    assert ws == 8 * 4096 * 8  # A = BS * K
    cq = moe.moe_combine_fwd_comm_quant_ws
    assert cq(s, *args2, 2, p, ctypes.c_void_p(264), ws, None) == moe.MOE_ERR_ALIGN
    assert cq(s, *args2, 2, p, p, ws - 1, None) == moe.MOE_ERR_CAPACITY
    assert cq(s, *args2, 2, p, p, ws, None) == moe.MOE_ERR_ARG  # ep_send_counts is NULL
    assert moe.moe_combine_bwd(s, None, p, None, p, p, None, p, p, None) == moe.MOE_ERR_ARG
    assert moe.moe_dispatch_bwd(s, p, None, None, p, None) == moe.MOE_ERR_ARG
    # special-expert backward: ori_x required; const tensors with const experts
    assert moe.moe_combine_bwd_special(ctypes.byref(sp.c()), p, p, p, None, None, p, p, p, p, p,
                                       p, p, p, p, 1 << 20, None) == moe.MOE_ERR_ARG
    assert moe.moe_combine_bwd_special(ctypes.byref(sp.c()), p, p, p, None, p, None, p, p, p, p,
                                       p, p, p, p, 1 << 20, None) == moe.MOE_ERR_ARG


def test_sizes():
    s = moe.Shape(bs=128, k=8, h=1536, num_experts=64)
    assert moe.moe_assist_info_elems(ctypes.byref(s.c())) == 1024 + 128 * 8
    assert moe.moe_layout_workspace_bytes(ctypes.byref(s.c())) == 0  # cluster layout
    # the cluster layout takes up to 16384 tokens while its masks and pair lists fit in
    # shared memory
    for bs, e, need_ws in ((16384, 256, False), (16385, 64, True), (8192, 512, False),
                           (8192, 1024, True)):
        sh = moe.Shape(bs=bs, k=8, h=1536, num_experts=e)
        assert (moe.moe_layout_workspace_bytes(ctypes.byref(sh.c())) > 0) == need_ws
    assert moe.moe_status_string(moe.MOE_ERR_CUDA) == b"CUDA error"


def test_tensor_wrappers_refuse_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        moe.dispatch_layout(moe.Shape(bs=4, k=2, h=1024, num_experts=4),
                            torch.zeros(4, 2, dtype=torch.int32),
                            workspace=torch.zeros(16, dtype=torch.uint8))
