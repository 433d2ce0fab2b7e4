"""The bounded waits of the staged kernels, made to run out on purpose through the
library's test hooks: one unit of work has its barrier armed for 16 bytes that no
copy delivers (so no copy is in flight for it), and the pipeline waits get a limit
of a few milliseconds. The call must return, the giving-up block (or warp) must be
counted once, everything it did write must be right, and the next ordinary call
must match the oracle bit for bit. No fault, trap or endless wait is involved."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workloads  # noqa: E402

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def test_int8_combine_gives_up_and_recovers():
    """The one-pass int8 combine (staged rows, producer warp + consumer warps)."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    wl = workloads.BY_NAME["special_int8_bs8192_h2048_k8_n70"].scaled(
        bs=1500, quant_mode=0, expert="identity", name="wait_test")
    inp = workloads.generate(wl)
    dt = wl.dtype
    _, send, assist, _ = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                wl.a_capacity)
    rng = np.random.default_rng(4)
    y = workloads.encode16(rng.standard_normal((wl.a_capacity, wl.h)), dt)
    want = oracle.combine_fwd(y, inp["topk_idx"], inp["topk_weights"], assist,
                              num_experts=wl.num_experts, a_capacity=wl.a_capacity, dtype=dt,
                              zero_expert_num=wl.zero_expert_num,
                              copy_expert_num=wl.copy_expert_num,
                              const_expert_num=wl.const_expert_num, ori_x=inp["ori_x"],
                              alpha1=inp["alpha1"], alpha2=inp["alpha2"], const_v=inp["v"],
                              comm_quant_mode=2)
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    idx, w = dev(inp["topk_idx"]), dev(inp["topk_weights"])
    lay = moe.dispatch_layout(sh, idx)
    y_d = dev(y, dt)
    ori, a1, a2, v = (dev(inp[k], dt) for k in ("ori_x", "alpha1", "alpha2", "v"))
    out = torch.full((wl.bs, wl.h), float("nan"), dtype=y_d.dtype, device=y_d.device)
    before = moe.moe_async_wait_timeouts()
    st = moe.moe_test_combine_fwd_comm_quant_wait_timeout(
        ctypes.byref(sh.c()), y_d.data_ptr(), idx.data_ptr(), w.data_ptr(),
        lay.assist_info.data_ptr(), None, None, ori.data_ptr(), a1.data_ptr(), a2.data_ptr(),
        v.data_ptr(), out.data_ptr(), LIMIT_NS, 1, _stream())
    assert st == moe.MOE_OK, moe.moe_status_string(st)
    torch.cuda.synchronize()
    assert moe.moe_async_wait_timeouts() == before + 1  # one block gave up
    got = host(out)
    done = ~np.isnan(workloads.decode16(got, dt)).any(axis=1)
    assert np.array_equal(got[done], want[done])  # what was written is right
    assert 0 < (~done).sum() < wl.bs // 2  # the block that gave up left its tokens
    # an ordinary call afterwards: bit for bit, and no new timeout
    out2 = moe.combine_fwd(sh, y_d, idx, w, lay, ori_x=ori, const_alpha_1=a1, const_alpha_2=a2,
                           const_v=v, comm_quant_mode=2, use_workspace=False)
    torch.cuda.synchronize()
    assert np.array_equal(host(out2), want)
    assert moe.moe_async_wait_timeouts() == before + 1


def test_smooth_dispatch_gives_up_and_recovers():
    """The smooth-scaled int8 dispatch (per-warp staged token rows)."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    wl = workloads.BY_NAME["special_int8_bs8192_h2048_k8_n70"].scaled(bs=1500, name="wait_test")
    inp = workloads.generate(wl)
    sm = workloads.smooth_scales(wl)
    _, send, assist, _ = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                wl.a_capacity)
    r = int(send[-1])
    q, s = oracle.dispatch_permute_quant_smooth(inp["x"], inp["topk_idx"], sm, assist,
                                                wl.a_capacity, wl.dtype)
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    idx = dev(inp["topk_idx"])
    lay = moe.dispatch_layout(sh, idx)
    x, sm_d = dev(inp["x"], wl.dtype), dev(sm)
    codes = torch.zeros((wl.a_capacity, wl.h), dtype=torch.int8, device=x.device)
    scales = torch.full((wl.a_capacity,), float("nan"), dtype=torch.float32, device=x.device)
    before = moe.moe_async_wait_timeouts()
    st = moe.moe_test_dispatch_permute_smooth_wait_timeout(
        ctypes.byref(sh.c()), x.data_ptr(), idx.data_ptr(), lay.assist_info.data_ptr(),
        lay.ep_send_counts.data_ptr(), sm_d.data_ptr(), codes.data_ptr(), scales.data_ptr(),
        LIMIT_NS, 0, _stream())
    assert st == moe.MOE_OK, moe.moe_status_string(st)
    torch.cuda.synchronize()
    assert moe.moe_async_wait_timeouts() == before + 1  # the first warp gave up
    got_s = host(scales)[:r]
    done = ~np.isnan(got_s)
    assert np.array_equal(host(codes)[:r][done], q[:r][done])
    assert np.array_equal(got_s[done].view(np.uint32), s[:r][done].view(np.uint32))
    assert 0 < (~done).sum() < r // 2
    qd, sd = moe.dispatch_permute_smooth(sh, x, idx, lay, sm_d)
    torch.cuda.synchronize()
    assert np.array_equal(host(qd)[:r], q[:r])
    assert np.array_equal(host(sd)[:r].view(np.uint32), s[:r].view(np.uint32))
    assert moe.moe_async_wait_timeouts() == before + 1


def test_hooks_refuse_bad_arguments():
    import combine_moe_dispatch_04_b200 as moe

    sh = moe.Shape(bs=64, k=8, h=2048, num_experts=64)
    p = ctypes.c_void_p(256)
    hook = moe.moe_test_dispatch_permute_smooth_wait_timeout
    args = [p] * 7
    assert hook(ctypes.byref(sh.c()), *args, 0, 0, None) == moe.MOE_ERR_ARG  # no limit
    assert hook(ctypes.byref(sh.c()), *args, 2 * 10**9, 0, None) == moe.MOE_ERR_ARG
    assert hook(ctypes.byref(sh.c()), *args, LIMIT_NS, -1, None) == moe.MOE_ERR_ARG
    k16 = moe.Shape(bs=64, k=16, h=1024, num_experts=64)  # K > 8: the other int8 combine
    cq = moe.moe_test_combine_fwd_comm_quant_wait_timeout
    assert cq(ctypes.byref(k16.c()), p, p, p, p, None, None, None, None, None, None, p, LIMIT_NS,
              0, None) == moe.MOE_ERR_UNSUPPORTED
