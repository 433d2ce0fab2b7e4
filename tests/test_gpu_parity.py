"""GPU parity: every kernel, called through the C ABI, against the CPU oracle on the
same seeded inputs. Bit-exact for layout, counts, assist_info, permuted rows and int8
codes/scales; 16-bit outputs within one ulp; grad_w within 1e-5 relative to
max(|grad_w|, sum_h |grad_out * expand_x|)."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workloads  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _chain():
    import gpu_chain
    return gpu_chain


W = {w.name.split("_")[0]: w for w in workloads.WORKLOADS}

# Reduced sizes that keep each workload's routing, dtype, masks and specials, span
# several layout tiles with a ragged tail, and exercise both layout paths
# (one CTA for BS <= 1024, tiled above).
SMALL = [
    W["tiny"],
    W["tiny"].scaled(bs=1000, h=1032, name="tiny_ragged"),
    W["uniform"].scaled(bs=2900, h=520, name="uniform_small"),
    W["uniform"].scaled(bs=777, h=1536, name="uniform_onecta"),
    W["dsv3"].scaled(bs=1333, h=896, name="dsv3_small"),
    W["mixtral"].scaled(bs=3001, h=264, name="mixtral_small"),
    W["mixtral"].scaled(bs=900, h=264, name="mixtral_onecta"),
    W["special"].scaled(bs=2100, h=1040, name="special_small"),
    W["special"].scaled(bs=515, h=2048, name="special_onecta"),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_parity(wl):
    rep = _chain().run_compare(workloads.generate(wl), twice=True)
    assert rep["combine_exact"] == 1.0, rep  # fp32 order matches: expected bit-exact


@pytest.mark.parametrize("wl", workloads.WORKLOADS, ids=lambda w: w.name)
def test_full_size_parity(wl):
    rep = _chain().run_compare(workloads.generate(wl))
    assert rep["combine_exact"] == 1.0, rep


def _custom(name, **kw):
    base = dict(name=name, bs=64, h=64, k=4, num_experts=16, backward=True, seed=99)
    base.update(kw)
    return workloads.Workload(**base)


EDGE = [
    _custom("empty", bs=0),
    _custom("one_token_k1", bs=1, k=1, num_experts=1),
    _custom("k16_e1024", bs=1500, k=16, num_experts=1024, h=128),
    _custom("k16_e1024_onecta", bs=300, k=16, num_experts=1024, h=128),
    _custom("mask1d", bs=1100, mask_ndim=1, mask_false_p=0.3),
    _custom("mask1d_onecta", bs=200, mask_ndim=1, mask_false_p=0.3),
    _custom("all_masked", bs=1200, mask_ndim=2, mask_false_p=1.0),
    _custom("spare_capacity", bs=1050, a_capacity_override=1050 * 4 + 777),
    _custom("min_h", bs=130, h=8),
    _custom("fp16_special", bs=1030, dtype="fp16", zero_expert_num=1, copy_expert_num=2,
            const_expert_num=3, backward=False),
    _custom("fp16_quant", bs=1030, h=2064, dtype="fp16", quant_mode=2, expert="dequant",
            backward=False),
    _custom("zipf_hot", bs=2048, k=2, num_experts=300, routing="zipf", zipf_s=3.0),
    # layout paths: the cluster kernel with 16 blocks of 512 and of 1024 threads (its
    # totals pushed to every block, or, at E = 512 with K = 16 where 16 x 513 totals do
    # not fit the pair-list area, loaded after the barrier; its slot -> pair entries
    # written per list entry, or, at E = 700 with K = 6 where the expert list does not
    # fit, per expert run), then the tiled count / column-scan / scatter path where the
    # cluster's shared memory does not suffice, just above its token limit, and at
    # 65536 tokens with E = 1024
    _custom("cluster16_e512_k16", bs=8192, k=16, num_experts=512, h=64),
    _custom("cluster_e700_1024_threads", bs=1500, k=4, num_experts=700, h=64),
    _custom("cluster_runs_e700_k6", bs=1500, k=6, num_experts=700, h=64),
    _custom("cluster_1024_threads", bs=16384, k=8, num_experts=256, h=64, mask_ndim=1,
            mask_false_p=0.2, backward=False),
    _custom("tiled_k16_e1024", bs=12000, k=16, num_experts=1024, h=64),
    _custom("tiled_just_above_cluster", bs=16385, k=4, num_experts=64, h=64, backward=False),
    _custom("tiled_bs65536_e1024", bs=65536, k=8, num_experts=1024, h=64, backward=False),
]


@pytest.mark.parametrize("wl", EDGE, ids=lambda w: w.name)
def test_edge_cases(wl):
    _chain().run_compare(workloads.generate(wl))


@pytest.mark.parametrize("bs", [600, 1800])
def test_invalid_ids_flagged_and_ignored(bs):
    wl = _custom("invalid_ids", bs=bs, k=4, num_experts=8, zero_expert_num=1, copy_expert_num=1,
                 const_expert_num=1)
    inp = workloads.generate(wl)
    idx = inp["topk_idx"].copy()
    idx[3, 2] = -5                 # below range
    idx[7, 0] = wl.n_ids + 3       # above range
    idx[11, 3] = idx[11, 1]        # repeat in a row
    idx[bs - 1, 1] = idx[bs - 1, 0]
    inp["topk_idx"] = idx
    inp["ori_x"] = inp["x"]
    _chain().run_compare(inp)


def test_all_tokens_one_expert():
    wl = _custom("one_expert", bs=2500, k=1, num_experts=4)
    inp = workloads.generate(wl)
    inp["topk_idx"] = np.full((wl.bs, 1), 2, np.int32)
    _chain().run_compare(inp)


COMM_QUANT = [
    W["special"].scaled(bs=1500, h=1040, name="special_q8"),
    W["uniform"].scaled(bs=2100, h=520, name="uniform_q8"),
    W["mixtral"].scaled(bs=1200, h=264, name="mixtral_fp16_mask_q8"),
    W["dsv3"].scaled(bs=300, h=7168, name="dsv3_shared_q8"),
    W["dsv3"].scaled(bs=300, h=1024, name="dsv3_shared_q8_staged"),  # shared add, staged
    _custom("k16_q8", bs=700, k=16, num_experts=40, h=136, zero_expert_num=2,
            const_expert_num=2, backward=False),
    _custom("zero_only_q8", bs=900, k=4, num_experts=16, zero_expert_num=3, h=256,
            backward=False),
    # routed pairs only: every K bucket of the two-pass gather, and rows too narrow for it
    _custom("k4_routed_q8", bs=700, k=4, num_experts=16, h=520, backward=False),
    _custom("k16_routed_q8", bs=600, k=16, num_experts=40, h=264, dtype="fp16",
            mask_ndim=2, mask_false_p=0.2, backward=False),
    _custom("k8_narrow_q8", bs=500, k=8, num_experts=32, h=136, backward=False),
    # special experts at H 3072: the single-pass kernel with two row buffers
    _custom("k8_h3072_special_q8", bs=300, k=8, num_experts=16, zero_expert_num=1,
            copy_expert_num=1, h=3072, backward=False),
    W["special"],  # full size
]


@pytest.mark.parametrize("use_ws", [True, False], ids=["two_pass", "single_pass"])
@pytest.mark.parametrize("wl", COMM_QUANT, ids=lambda w: w.name)
def test_combine_comm_quant_mode2(wl, use_ws):
    """Combine with comm_quant_mode 2 (per-row int8 round trip of the returning
    rows) against the oracle on the same expert outputs, with and without the
    workspace (two-pass kernels where the shape allows, else the single pass)."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    inp = workloads.generate(wl)
    dt = wl.dtype
    _, send, assist, st = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                 wl.a_capacity, inp["mask"])
    rng = np.random.default_rng(5)
    y = workloads.encode16(rng.standard_normal((wl.a_capacity, wl.h)) *
                           rng.uniform(0.01, 10, (wl.a_capacity, 1)), dt)
    y[:3] = 0  # all-zero rows: scale 0
    want = oracle.combine_fwd(y, inp["topk_idx"], inp["topk_weights"], assist,
                              num_experts=wl.num_experts, a_capacity=wl.a_capacity, dtype=dt,
                              zero_expert_num=wl.zero_expert_num,
                              copy_expert_num=wl.copy_expert_num,
                              const_expert_num=wl.const_expert_num, mask=inp["mask"],
                              shared=inp["shared"], ori_x=inp["ori_x"], alpha1=inp["alpha1"],
                              alpha2=inp["alpha2"], const_v=inp["v"], comm_quant_mode=2)
    sh = gpu_chain.shape_of(wl)
    dev = gpu_chain.dev
    lay = moe.dispatch_layout(sh, dev(inp["topk_idx"]), dev(inp["mask"]))
    out = moe.combine_fwd(sh, dev(y, dt), dev(inp["topk_idx"]), dev(inp["topk_weights"]), lay,
                          x_active_mask=dev(inp["mask"]), shared_expert_x=dev(inp["shared"], dt),
                          ori_x=dev(inp["ori_x"], dt), const_alpha_1=dev(inp["alpha1"], dt),
                          const_alpha_2=dev(inp["alpha2"], dt), const_v=dev(inp["v"], dt),
                          comm_quant_mode=2, use_workspace=use_ws)
    torch.cuda.synchronize()
    got = gpu_chain.host(out)
    d = gpu_chain.ulp_dist(got, want)
    assert d.max() <= gpu_chain.ULP_TOL
    assert (d == 0).mean() == 1.0  # same fp32 operations in the same order
    assert moe.moe_async_wait_timeouts() == 0  # no staged copy was given up on


@pytest.mark.parametrize("use_ws", [True, False], ids=["two_pass", "single_pass"])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_combine_q8_rounding_ties(dtype, use_ws):
    """Returning rows whose values sit exactly on, or one 16-bit step beside,
    half-integer multiples of their scale: the combine round trip must match the
    oracle's IEEE division and rounding bit for bit. With the workspace the shape is
    one the two-pass kernels take (routed pairs only, H / 8 >= 32 U); in bf16 some
    rows have scales below 2^-100, which take the IEEE-division branch."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    k, h = (8, 256) if use_ws else (4, 256)
    wl = _custom("q8_ties", bs=600, k=k, num_experts=16, h=h, backward=False, dtype=dtype)
    u = 4 if k <= 2 else 2 if k <= 4 else 1
    assert (h // 8 >= 32 * u) == use_ws  # the two-pass kernels' condition
    inp = workloads.generate(wl)
    _, send, assist, st = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                 wl.a_capacity)
    rng = np.random.default_rng(23)
    a_rows = wl.a_capacity
    c = 2.0 ** rng.integers(-6, 3, (a_rows, 1))
    if dtype == "bf16":  # scales 2^-110 .. 2^-102: below the reciprocal's range
        tiny = rng.random(a_rows) < 0.1
        c[tiny, 0] = 2.0 ** rng.integers(-110, -101, int(tiny.sum()))
    ties = (rng.integers(-127, 127, (a_rows, wl.h)) + 0.5) * c
    ties[:, 0] = 127 * c[:, 0]  # the row max, so scale = c exactly
    y = workloads.encode16(ties, dtype)
    step = rng.integers(-1, 2, y.shape).astype(np.int32)
    step[:, 0] = 0
    y = (y.astype(np.int32) + step * (rng.random(y.shape) < 0.3)).astype(np.uint16)
    want = oracle.combine_fwd(y, inp["topk_idx"], inp["topk_weights"], assist,
                              num_experts=wl.num_experts, a_capacity=wl.a_capacity, dtype=dtype,
                              comm_quant_mode=2)
    sh = gpu_chain.shape_of(wl)
    dev = gpu_chain.dev
    lay = moe.dispatch_layout(sh, dev(inp["topk_idx"]))
    out = moe.combine_fwd(sh, dev(y, dtype), dev(inp["topk_idx"]), dev(inp["topk_weights"]), lay,
                          comm_quant_mode=2, use_workspace=use_ws)
    torch.cuda.synchronize()
    assert np.array_equal(gpu_chain.host(out), want)


FUSED = [
    W["tiny"],
    _custom("fused_ragged", bs=1000, h=1032),
    _custom("fused_max", bs=1024, h=264, k=8, num_experts=64),
    _custom("fused_k16_e1024", bs=300, k=16, num_experts=1024, h=128),
    _custom("fused_mask1d", bs=700, mask_ndim=1, mask_false_p=0.3),
    _custom("fused_mask2d_fp16", bs=513, mask_ndim=2, mask_false_p=0.2, dtype="fp16"),
    _custom("fused_special", bs=600, zero_expert_num=1, copy_expert_num=1, const_expert_num=1),
    _custom("fused_empty", bs=0),
    _custom("fused_tiled_ragged", bs=2100, h=520),
    _custom("fused_tiled_k16_e1024", bs=1500, k=16, num_experts=1024, h=128),
    _custom("fused_tiled_one_tile_tail", bs=1025, h=64),
    W["uniform"],
    W["mixtral"],
    W["dsv3"].scaled(bs=3000, h=1024, name="fused_tiled_zipf"),
    W["special"].scaled(bs=800, h=1040, name="fused_fallback_int8"),
    W["special"].scaled(bs=2600, h=1040, quant_mode=0, name="fused_tiled_special"),
]


@pytest.mark.parametrize("wl", FUSED, ids=lambda w: w.name)
def test_fused_dispatch(wl):
    """moe_dispatch (layout + permute, one launch for small batches) against the
    oracle: counts, prefix sums, assist_info, status and every expanded row bit for
    bit; ids out of range and repeats are planted in the batches that have rows."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    inp = workloads.generate(wl)
    if wl.bs > 20:
        idx = inp["topk_idx"].copy()
        idx[5, 0] = -3
        idx[9, wl.k - 1] = idx[9, 0]
        inp["topk_idx"] = idx
    counts, send, assist, status = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts,
                                                          wl.n_ids, wl.a_capacity, inp["mask"])
    r = int(send[-1])
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    lay, ex, sc = moe.dispatch(sh, dev(inp["topk_idx"]), dev(inp["x"], wl.dtype),
                               x_active_mask=dev(inp["mask"]), comm_quant_mode=wl.quant_mode)
    torch.cuda.synchronize()
    assert np.array_equal(host(lay.expert_token_nums), counts)
    assert np.array_equal(host(lay.ep_send_counts), send)
    assert np.array_equal(host(lay.assist_info), assist)
    assert int(host(lay.dev_status)[0]) & 3 == status
    if wl.quant_mode == 2:
        q, s = oracle.dispatch_permute_quant(inp["x"], assist, wl.k, wl.a_capacity, wl.dtype)
        assert np.array_equal(host(ex)[:r], q[:r])
        assert np.array_equal(host(sc)[:r].view(np.uint32), s[:r].view(np.uint32))
    else:
        want = oracle.dispatch_permute(inp["x"], assist, wl.k, wl.a_capacity)
        assert np.array_equal(host(ex)[:r], want[:r])


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_int8_quant_rounding_ties(dtype):
    """Rows whose quotients x / scale are exact half-integers (ties, decided by
    round-half-even) or lie next to them: the kernel's quantisation must match the
    oracle's IEEE division and rounding code for code."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe
    from golden_io import read

    h = 64
    rows = []
    g = read("quant_rows.txt")
    for r in g["x"]:
        rows.append(np.pad(np.array(r, np.float64), (0, h - len(r))))
    rng = np.random.default_rng(17)
    for amax in (127.0, 63.5, 31.75, 100.0, 3.0, 0.01):
        ties = (rng.integers(-126, 126, h) + 0.5) * (amax / 127.0)
        ties[0] = amax
        rows.append(ties)
        near = ties * (1 + rng.choice([-1, 1], h) * rng.uniform(0, 4e-3, h))
        near[0] = amax
        rows.append(near)
    x = workloads.encode16(np.array(rows), dtype)
    bs = len(rows)
    idx = np.zeros((bs, 1), np.int32)
    _, send, assist, _ = oracle.dispatch_layout(idx, 1, 1, bs)
    q, sc = oracle.dispatch_permute_quant(x, assist, 1, bs, dtype)
    sh = moe.Shape(bs=bs, k=1, h=h, num_experts=1, dtype=workloads.DTYPE_CODES[dtype])
    lay = moe.dispatch_layout(sh, gpu_chain.dev(idx))
    qd, scd = moe.dispatch_permute(sh, gpu_chain.dev(x, dtype), lay, 2)
    torch.cuda.synchronize()
    assert np.array_equal(gpu_chain.host(qd), q)
    assert np.array_equal(gpu_chain.host(scd).view(np.uint32), sc.view(np.uint32))


SMOOTH = [
    W["special"],
    W["special"].scaled(bs=1500, h=528, mask_ndim=2, mask_false_p=0.2, name="special_mask"),
    W["dsv3"].scaled(bs=700, dtype="fp16", name="dsv3_fp16"),  # rows streamed twice
    _custom("smooth_h16384", bs=40, k=3, num_experts=5, h=16384, quant_mode=2),
    _custom("smooth_h4096", bs=200, k=4, num_experts=8, h=4096, quant_mode=2),  # 4 warps
    _custom("smooth_h16_one_expert", bs=333, k=1, num_experts=1, h=16, quant_mode=2),
    _custom("smooth_empty", bs=0, quant_mode=2),
]


@pytest.mark.parametrize("wl", SMOOTH, ids=lambda w: w.name)
def test_dispatch_smooth_quant(wl):
    """int8 dispatch of x[t] * smooth[e]: codes and scales bit for bit against the
    oracle; with several experts, expert 0's factors are zero, so its rows give
    scale 0 and zero codes."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    inp = workloads.generate(wl)
    sm = workloads.smooth_scales(wl)
    if wl.num_experts > 1:
        sm[0] = 0.0
    _, send, assist, _ = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                wl.a_capacity, mask=inp["mask"])
    r = int(send[-1])
    q, s = oracle.dispatch_permute_quant_smooth(inp["x"], inp["topk_idx"], sm, assist,
                                                wl.a_capacity, wl.dtype)
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    idx = dev(inp["topk_idx"])
    lay = moe.dispatch_layout(sh, idx, x_active_mask=dev(inp["mask"]))
    qd, sd = moe.dispatch_permute_smooth(sh, dev(inp["x"], wl.dtype), idx, lay, dev(sm))
    torch.cuda.synchronize()
    assert np.array_equal(host(qd)[:r], q[:r])
    assert np.array_equal(host(sd)[:r].view(np.uint32), s[:r].view(np.uint32))


SPECIAL_BWD = [
    W["special"].scaled(backward=True, name="special_full_bwd"),
    W["special"].scaled(bs=1500, h=520, backward=True, mask_ndim=2, mask_false_p=0.2,
                        name="special_mask_bwd"),
    _custom("special_fp16_k16_bwd", bs=900, k=16, num_experts=24, zero_expert_num=2,
            copy_expert_num=3, const_expert_num=4, h=264, dtype="fp16"),
    _custom("special_copy_only_bwd", bs=700, k=4, num_experts=8, copy_expert_num=2, h=136),
]


@pytest.mark.parametrize("wl", SPECIAL_BWD, ids=lambda w: w.name)
def test_special_expert_backward(wl):
    """Backward through the copy/const experts against the oracle: grad_w of those
    pairs within 1e-5 of max(|ref|, sum |terms|), grad_ori_x within one ulp, and the
    alpha / v gradients within 1e-5 of their sums of |terms|."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    inp = workloads.generate(wl)
    inp["ori_x"] = inp["x"]
    dt = wl.dtype
    ref = oracle.combine_bwd_special(
        inp["grad_out"], inp["topk_idx"], inp["topk_weights"], num_experts=wl.num_experts,
        dtype=dt, zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
        const_expert_num=wl.const_expert_num, mask=inp["mask"], ori_x=inp["ori_x"],
        alpha1=inp["alpha1"], alpha2=inp["alpha2"], const_v=inp["v"])
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    gw, gox, ga1, ga2, gv = moe.combine_bwd_special(
        sh, dev(inp["grad_out"], dt), dev(inp["topk_idx"]), dev(inp["topk_weights"]),
        dev(inp["x"], dt), x_active_mask=dev(inp["mask"]), const_alpha_1=dev(inp["alpha1"], dt),
        const_alpha_2=dev(inp["alpha2"], dt), const_v=dev(inp["v"], dt))
    torch.cuda.synchronize()

    def close(got, want, mag, name):
        err = np.abs(got.astype(np.float64) - want.astype(np.float64))
        bound = 1e-5 * np.maximum(np.abs(want.astype(np.float64)), mag)
        assert np.all(err <= bound), (name, float((err / np.maximum(bound, 1e-30)).max()))

    close(host(gw), ref["grad_w"], ref["abs_sum"], "grad_w")
    d = gpu_chain.ulp_dist(host(gox), ref["grad_ori_x"])
    assert d.max() <= 1 and (d == 0).mean() == 1.0
    if wl.const_expert_num:
        close(host(ga1), ref["grad_alpha1"], ref["abs_alpha1"], "grad_alpha1")
        close(host(ga2), ref["grad_alpha2"], ref["abs_alpha2"], "grad_alpha2")
        close(host(gv), ref["grad_v"], ref["abs_v"], "grad_v")


QBWD = [
    W["special"].scaled(backward=True, name="special_full_q8_bwd"),
    W["uniform"].scaled(name="uniform_full_q8_bwd"),
    W["mixtral"].scaled(bs=1200, h=264, name="mixtral_fp16_mask_q8_bwd"),
    _custom("k16_narrow_q8_bwd", bs=700, k=16, num_experts=40, h=136),
]


@pytest.mark.parametrize("wl", QBWD, ids=lambda w: w.name)
def test_combine_bwd_comm_quant_mode2(wl):
    """Backward of the int8 round-trip combine against the oracle: grad_expand bit
    for bit (the round trip passed straight through), grad_w within 1e-5 of
    max(|ref|, sum_h |grad_out * D(y)|), D the round-trip values; rows include
    all-zero rows and, in bf16, rows whose scale is below 2^-100."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    inp = workloads.generate(wl)
    dt = wl.dtype
    _, send, assist, st = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                 wl.a_capacity, inp["mask"])
    r = int(send[-1])
    rng = np.random.default_rng(9)
    scale = rng.uniform(0.01, 10, (wl.a_capacity, 1))
    if dt == "bf16":
        scale[rng.random(wl.a_capacity) < 0.05] = 2.0 ** -110
    y = workloads.encode16(rng.standard_normal((wl.a_capacity, wl.h)) * scale, dt)
    y[:3] = 0
    ge_ref, gw_ref, mag = oracle.combine_bwd(inp["grad_out"], y, inp["topk_weights"], assist,
                                             k=wl.k, a_capacity=wl.a_capacity, dtype=dt,
                                             mask=inp["mask"], comm_quant_mode=2)
    sh = gpu_chain.shape_of(wl)
    dev, host = gpu_chain.dev, gpu_chain.host
    lay = moe.dispatch_layout(sh, dev(inp["topk_idx"]), dev(inp["mask"]))
    ge, gw = moe.combine_bwd(sh, dev(inp["grad_out"], dt), dev(y, dt), dev(inp["topk_weights"]),
                             lay, x_active_mask=dev(inp["mask"]), comm_quant_mode=2)
    torch.cuda.synchronize()
    assert np.array_equal(host(ge)[:r], ge_ref[:r])
    err = np.abs(host(gw).astype(np.float64) - gw_ref.astype(np.float64))
    bound = gpu_chain.GRAD_W_RTOL * np.maximum(np.abs(gw_ref.astype(np.float64)), mag)
    assert np.all(err <= bound), float((err / np.maximum(bound, 1e-30)).max())


@pytest.mark.parametrize("k", [8, 2])
def test_combine_ignores_weights_of_skipped_pairs(k):
    """Masked pairs, invalid and repeated ids carry NaN weights: combine must
    leave them out exactly as the oracle does (the K > 4 gather sums a skipped
    pair as a zero vector with weight 0, so the weight it holds never enters)."""
    import gpu_chain
    import oracle
    import combine_moe_dispatch_04_b200 as moe

    wl = _custom(f"nan_skip_k{k}", bs=900, k=k, num_experts=32, h=256, mask_ndim=2,
                 mask_false_p=0.3, backward=False)
    inp = workloads.generate(wl)
    idx = inp["topk_idx"].copy()
    idx[::7, 0] = wl.num_experts + 5      # out of range
    idx[1::11, k - 1] = idx[1::11, 0]     # a repeat of the token's first id
    w = inp["topk_weights"].copy()
    skipped = (inp["mask"] == 0)
    skipped[::7, 0] = True
    skipped[1::11, k - 1] = True
    w[skipped] = np.nan
    _, send, assist, _ = oracle.dispatch_layout(idx, wl.num_experts, wl.n_ids, wl.a_capacity,
                                                inp["mask"])
    rng = np.random.default_rng(5)
    y = workloads.encode16(rng.standard_normal((wl.a_capacity, wl.h)), wl.dtype)
    want = oracle.combine_fwd(y, idx, w, assist, num_experts=wl.num_experts,
                              a_capacity=wl.a_capacity, dtype=wl.dtype, mask=inp["mask"])
    assert not np.isnan(workloads.decode16(want, wl.dtype)).any()
    sh = gpu_chain.shape_of(wl)
    idx_d, mask_d = gpu_chain.dev(idx), gpu_chain.dev(inp["mask"])
    lay = moe.dispatch_layout(sh, idx_d, mask_d)
    out = moe.combine_fwd(sh, gpu_chain.dev(y, wl.dtype), idx_d, gpu_chain.dev(w), lay,
                          x_active_mask=mask_d)
    torch.cuda.synchronize()
    assert np.array_equal(gpu_chain.host(out), want)
