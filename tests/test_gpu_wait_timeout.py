"""The bounded waits of the staged kernels, made to run out on purpose through the
library's test hooks: one unit of work has its barrier armed for 16 bytes that no
copy delivers (so no copy is in flight for it), and the pipeline waits get a limit
of a few milliseconds. The call must return, the giving-up block must be counted
once, the rest of the output must be right, and the next ordinary call must match
the oracle bit for bit. No fault, trap or endless wait is involved."""
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


@pytest.mark.parametrize("special", [False, True])
def test_staged_combine_gives_up_and_recovers(special):
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    base = workloads.BY_NAME["special_int8_bs8192_h2048_k8_n70" if special
                             else "uniform_bs8192_h1536_k8_e64"]
    wl = base.scaled(bs=1500, quant_mode=0, expert="identity", name="wait_test")
    inp = workloads.generate(wl)
    dt = wl.dtype
    _, send, assist, _ = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                wl.a_capacity)
    rng = np.random.default_rng(4)
    y = workloads.encode16(rng.standard_normal((wl.a_capacity, wl.h)), dt)
    kw = dict(num_experts=wl.num_experts, a_capacity=wl.a_capacity, dtype=dt,
              zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
              const_expert_num=wl.const_expert_num, ori_x=inp["ori_x"], alpha1=inp["alpha1"],
              alpha2=inp["alpha2"], const_v=inp["v"])
    want = oracle.combine_fwd(y, inp["topk_idx"], inp["topk_weights"], assist, **kw)
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    idx, w = dev(inp["topk_idx"]), dev(inp["topk_weights"])
    lay = moe.dispatch_layout(sh, idx)
    y_d = dev(y, dt)
    extra = [dev(inp[k], dt) for k in ("ori_x", "alpha1", "alpha2", "v")]
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    sentinel = torch.full((wl.bs, wl.h), float("nan"), dtype=y_d.dtype, device=y_d.device)
    before = moe.moe_async_wait_timeouts()
    st = moe.moe_test_combine_fwd_wait_timeout(
        ctypes.byref(sh.c()), y_d.data_ptr(), idx.data_ptr(), w.data_ptr(),
        lay.assist_info.data_ptr(), None, None, *[ptr(t) for t in extra], sentinel.data_ptr(),
        LIMIT_NS, 1, _stream())
    assert st == moe.MOE_OK, moe.moe_status_string(st)
    torch.cuda.synchronize()
    assert moe.moe_async_wait_timeouts() == before + 1  # one block gave up
    got = host(sentinel)
    done = ~np.isnan(workloads.decode16(got, dt)).any(axis=1)
    assert np.array_equal(got[done], want[done])  # what was written is right
    assert 0 < (~done).sum() < wl.bs // 2  # the block that gave up left its tokens
    # an ordinary call afterwards: bit for bit, and no new timeout
    out = moe.combine_fwd(sh, y_d, idx, w, lay, ori_x=extra[0], const_alpha_1=extra[1],
                          const_alpha_2=extra[2], const_v=extra[3])
    torch.cuda.synchronize()
    assert np.array_equal(host(out), want)
    assert moe.moe_async_wait_timeouts() == before + 1


def test_bulk_permute_gives_up_and_recovers():
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    wl = workloads.BY_NAME["uniform_bs8192_h1536_k8_e64"].scaled(bs=3000, name="wait_test")
    inp = workloads.generate(wl)
    _, send, assist, _ = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                wl.a_capacity)
    r = int(send[-1])
    want = oracle.dispatch_permute(inp["x"], assist, wl.k, wl.a_capacity)
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    lay = moe.dispatch_layout(sh, dev(inp["topk_idx"]))
    x = dev(inp["x"], wl.dtype)
    ex = torch.zeros((wl.a_capacity, wl.h), dtype=x.dtype, device=x.device)
    before = moe.moe_async_wait_timeouts()
    st = moe.moe_test_dispatch_permute_wait_timeout(
        ctypes.byref(sh.c()), x.data_ptr(), lay.assist_info.data_ptr(), ex.data_ptr(), LIMIT_NS,
        0, _stream())
    assert st == moe.MOE_OK, moe.moe_status_string(st)
    torch.cuda.synchronize()
    assert moe.moe_async_wait_timeouts() == before + 1  # the first warp gave up
    got = host(ex)[:r]
    written = (got != 0).any(axis=1)
    assert np.array_equal(got[written], want[:r][written])
    assert 0 < (~written).sum() < r // 2
    ex2, _ = moe.dispatch_permute(sh, x, lay, 0)
    torch.cuda.synchronize()
    assert np.array_equal(host(ex2)[:r], want[:r])
    assert moe.moe_async_wait_timeouts() == before + 1


def test_hooks_refuse_bad_arguments():
    import combine_moe_dispatch_04_b200 as moe

    sh = moe.Shape(bs=64, k=8, h=1536, num_experts=64)
    p = ctypes.c_void_p(256)
    hook = moe.moe_test_dispatch_permute_wait_timeout
    assert hook(ctypes.byref(sh.c()), p, p, p, 0, 0, None) == moe.MOE_ERR_ARG  # no limit
    assert hook(ctypes.byref(sh.c()), p, p, p, 2 * 10**9, 0, None) == moe.MOE_ERR_ARG
    assert hook(ctypes.byref(sh.c()), p, p, p, LIMIT_NS, -1, None) == moe.MOE_ERR_ARG
    narrow = moe.Shape(bs=64, k=8, h=64, num_experts=64)  # rows for the register kernel
    assert hook(ctypes.byref(narrow.c()), p, p, p, LIMIT_NS, 0, None) == moe.MOE_ERR_UNSUPPORTED
