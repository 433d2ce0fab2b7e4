"""The allocation-free layout entry point, moe_dispatch_layout_noalloc.

Some callers cannot allocate device memory: code that runs inside a host framework
which owns every byte of device memory and gives its plugins no allocator, or a
latency-critical serving loop that must not call cudaMalloc (it can synchronise the
device). For them the layout uses a fixed scratch array compiled into the library
instead of a caller-provided workspace. This file checks, through the C ABI, that two
calls in a row give exactly what moe_dispatch_layout gives (the layout is compared
bit for bit, as everywhere in these tests), and that a shape too large for the fixed
array is refused before anything runs.

The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import combine_moe_dispatch_04_b200 as moe  # noqa: E402
import workloads  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _outputs(shape, dev):
    return moe.Layout(torch.full((shape.num_experts,), -7, dtype=torch.int32, device=dev),
                      torch.full((shape.num_experts + 1,), -7, dtype=torch.int32, device=dev),
                      torch.full((shape.A + shape.bs * shape.k,), -7, dtype=torch.int32,
                                 device=dev),
                      torch.full((1,), -7, dtype=torch.int32, device=dev))


def _host(lay):
    return [t.cpu().numpy() for t in (lay.expert_token_nums, lay.ep_send_counts,
                                      lay.assist_info, lay.dev_status)]


@pytest.mark.parametrize("wl", [
    workloads.WORKLOADS[1],                                      # 8192 tokens, tiled layout
    workloads.WORKLOADS[3],                                      # 16384 tokens, 2-D mask
    workloads.WORKLOADS[4].scaled(bs=3000, h=64),                # special experts
    workloads.WORKLOADS[0],                                      # 128 tokens, one-CTA layout
    # tiled layouts, the ones that use the scratch array
    workloads.WORKLOADS[1].scaled(bs=20000, h=64, name="tiled_20000"),
    workloads.WORKLOADS[2].scaled(bs=40000, h=64, name="tiled_40000_e256"),
], ids=lambda w: w.name)
def test_noalloc_matches_workspace_layout_twice(wl):
    dev = torch.device("cuda", 0)
    inp = workloads.generate(wl)
    sh = moe.Shape(bs=wl.bs, k=wl.k, h=wl.h, num_experts=wl.num_experts,
                   zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
                   const_expert_num=wl.const_expert_num, a_capacity=wl.a_capacity,
                   dtype=workloads.DTYPE_CODES[wl.dtype], mask_ndim=wl.mask_ndim)
    idx = torch.from_numpy(inp["topk_idx"]).to(dev)
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    want = _host(moe.dispatch_layout(sh, idx, mask))
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        out = _outputs(sh, dev)
        st = moe.moe_dispatch_layout_noalloc(
            ctypes.byref(sh.c()), idx.data_ptr(), None if mask is None else mask.data_ptr(),
            out.expert_token_nums.data_ptr(), out.ep_send_counts.data_ptr(),
            out.assist_info.data_ptr(), out.dev_status.data_ptr(),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == moe.MOE_OK, moe.moe_status_string(st)
        torch.cuda.synchronize()
        for g, w in zip(_host(out), want):
            assert np.array_equal(g, w)


def test_noalloc_refuses_shapes_beyond_its_scratch():
    limit = moe.moe_layout_noalloc_max_workspace_bytes()
    big = moe.Shape(bs=70000, k=16, h=1024, num_experts=1024)
    assert moe.moe_layout_workspace_bytes(ctypes.byref(big.c())) > limit
    # real buffers of the shape's sizes: were the size check ever lost, the layout
    # would run on valid memory and this assertion would fail, not the GPU
    dev = torch.device("cuda", 0)
    idx = torch.zeros((big.bs, big.k), dtype=torch.int32, device=dev)
    out = _outputs(big, dev)
    st = moe.moe_dispatch_layout_noalloc(
        ctypes.byref(big.c()), idx.data_ptr(), None, out.expert_token_nums.data_ptr(),
        out.ep_send_counts.data_ptr(), out.assist_info.data_ptr(), out.dev_status.data_ptr(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_ERR_CAPACITY
    torch.cuda.synchronize()
    assert int(out.ep_send_counts[0].item()) == -7  # nothing was written
