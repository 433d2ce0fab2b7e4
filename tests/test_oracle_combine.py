"""Pins of the oracle's combine forward, combine backward and dispatch backward:
hand-computed cases, rounding-order cases, closed forms of the special experts,
the exact float64 result within the fp32/bf16 rounding bound, and a
finite-difference gradient."""
import numpy as np
import pytest

import oracle
import workloads
from golden_io import read


def ulp_dist(a, b):
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordered(a) - ordered(b))


def _layout(idx, e, n, a_cap, mask=None):
    counts, send, assist, st = oracle.dispatch_layout(idx, e, n, a_cap, mask)
    assert st == 0
    return assist, int(send[-1])


def _hand_inputs(g):
    dt = g["dtype"]
    enc = lambda k: workloads.encode16(np.array(g[k], np.float32), dt)
    return dict(idx=np.array(g["topk_idx"], np.int32), w=np.array(g["topk_weights"], np.float32),
                x=enc("x"), a1=enc("alpha1"), a2=enc("alpha2"), v=enc("const_v"),
                shared=enc("shared"), mask=np.array(g["mask"], np.uint8))


@pytest.mark.parametrize("variant", ["out_no_shared", "out_shared", "out_masked_shared"])
def test_hand_case(variant):
    g = read("combine_hand.txt")
    d = _hand_inputs(g)
    e, z, c, q = (g["num_experts"], g["zero_expert_num"], g["copy_expert_num"],
                  g["const_expert_num"])
    mask = d["mask"] if variant == "out_masked_shared" else None
    bs, k = d["idx"].shape
    assist, r = _layout(d["idx"], e, e + z + c + q, bs * k, mask)
    assert r == (g["routed_masked_total"] if mask is not None else g["routed_total"])
    y = oracle.dispatch_permute(d["x"], assist, k, bs * k)
    out = oracle.combine_fwd(y, d["idx"], d["w"], assist, num_experts=e, a_capacity=bs * k,
                             dtype=g["dtype"], zero_expert_num=z, copy_expert_num=c,
                             const_expert_num=q, mask=mask,
                             shared=None if variant == "out_no_shared" else d["shared"],
                             ori_x=d["x"], alpha1=d["a1"], alpha2=d["a2"], const_v=d["v"])
    want = workloads.encode16(np.array(g[variant], np.float32), g["dtype"])
    assert np.array_equal(out, want)


@pytest.mark.parametrize("case", ["order", "no_fma"])
def test_rounding_cases(case):
    g = read("combine_rounding.txt")["cases"][case]
    k = len(g["w"])
    idx = np.arange(k, dtype=np.int32)[None, :]
    w = np.array([g["w"]], np.float32)
    assert w.astype(np.float64).tolist() == [g["w"]]  # weights exact in fp32
    assist, r = _layout(idx, k, k, k)
    y = workloads.encode16(np.array(g["m"], np.float32)[:, None], "bf16")  # slot k <- expert k
    out = oracle.combine_fwd(y, idx, w, assist, num_experts=k, a_capacity=k, dtype="bf16")
    assert workloads.decode16(out, "bf16")[0, 0] == np.float32(g["out"])


def _random_case(dtype, bs=40, h=24, k=4, e=6, z=1, c=1, q=1, seed=0, mask_ndim=0):
    rng = np.random.default_rng(seed)
    n = e + z + c + q
    idx = np.argsort(rng.random((bs, n)), axis=1)[:, :k].astype(np.int32)
    w = rng.uniform(-1, 1, (bs, k)).astype(np.float32)
    enc = lambda shape, s=1.0: workloads.encode16(rng.standard_normal(shape) * s, dtype)
    d = dict(idx=idx, w=w, x=enc((bs, h)), shared=enc((bs, h)), a1=enc((q, h)), a2=enc((q, h)),
             v=enc((q, h)), g=enc((bs, h)), e=e, z=z, c=c, q=q, n=n, bs=bs, h=h, k=k)
    d["mask"] = None
    if mask_ndim == 1:
        d["mask"] = (rng.random(bs) > 0.2).astype(np.uint8)
    elif mask_ndim == 2:
        d["mask"] = (rng.random((bs, k)) > 0.2).astype(np.uint8)
    d["assist"], d["r"] = _layout(idx, e, n, bs * k, d["mask"])
    d["y"] = workloads.encode16(rng.standard_normal((bs * k, h)), dtype)  # expert outputs
    return d


def _combine(d, dtype, **over):
    kw = dict(num_experts=d["e"], a_capacity=d["bs"] * d["k"], dtype=dtype,
              zero_expert_num=d["z"], copy_expert_num=d["c"], const_expert_num=d["q"],
              mask=d["mask"], shared=d["shared"], ori_x=d["x"], alpha1=d["a1"],
              alpha2=d["a2"], const_v=d["v"])
    kw.update(over)
    return oracle.combine_fwd(d["y"], d["idx"], d["w"], d["assist"], **kw)


def _exact_combine(d, dtype, with_shared=True):
    """Float64 value of the combine formula, before any rounding."""
    f = lambda a: workloads.decode16(a, dtype).astype(np.float64)
    x, y = f(d["x"]), f(d["y"])
    out = f(d["shared"]) if with_shared else np.zeros_like(x)
    e, z, c = d["e"], d["z"], d["c"]
    for t in range(d["bs"]):
        for kk in range(d["k"]):
            if d["mask"] is not None:
                act = d["mask"][t] if d["mask"].ndim == 1 else d["mask"][t, kk]
                if not act:
                    continue
            i = d["idx"][t, kk]
            wt = float(d["w"][t, kk])
            if i < e:
                out[t] += wt * y[d["assist"][d["bs"] * d["k"] + t * d["k"] + kk]]
            elif i < e + z:
                pass
            elif i < e + z + c:
                out[t] += wt * x[t]
            else:
                j = i - (e + z + c)
                out[t] += wt * (f(d["a1"])[j] * x[t] + f(d["a2"])[j] * f(d["v"])[j])
    return out


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("mask_ndim", [0, 1, 2])
def test_combine_within_rounding_of_exact(dtype, mask_ndim):
    d = _random_case(dtype, seed=mask_ndim, mask_ndim=mask_ndim)
    out = _combine(d, dtype)
    exact = workloads.encode16(_exact_combine(d, dtype), dtype)
    dist = ulp_dist(out, exact)
    assert dist.max() <= 1
    assert (dist == 0).mean() > 0.97


def test_special_expert_closed_forms():
    dtype = "bf16"
    d = _random_case(dtype, k=1, e=2, z=1, c=1, q=1, seed=5)
    bs, h = d["bs"], d["h"]
    ones = np.ones((bs, 1), np.float32)
    # zero expert only -> out = shared exactly, or 0 without shared
    d0 = dict(d, idx=np.full((bs, 1), 2, np.int32), w=ones)
    d0["assist"], _ = _layout(d0["idx"], 2, 5, bs)
    assert np.array_equal(_combine(d0, dtype), d["shared"])
    assert not _combine(d0, dtype, shared=None).any()
    # copy expert, weight 1 -> out = ori_x exactly
    d1 = dict(d0, idx=np.full((bs, 1), 3, np.int32))
    assert np.array_equal(_combine(d1, dtype, shared=None), d["x"])
    # const expert with alpha_1 = 1, alpha_2 = 0 is a copy expert
    one = workloads.encode16(np.ones((1, h)), dtype)
    zero = workloads.encode16(np.zeros((1, h)), dtype)
    d2 = dict(d0, idx=np.full((bs, 1), 4, np.int32))
    assert np.array_equal(_combine(d2, dtype, shared=None, alpha1=one, alpha2=zero), d["x"])
    # const expert with alpha_1 = 0, alpha_2 = 1 returns v for every token
    assert np.array_equal(_combine(d2, dtype, shared=None, alpha1=zero, alpha2=one),
                          np.repeat(d["v"], bs, axis=0))
    # routed expert, weight 1, K = 1: dispatch then combine is the identity
    d3 = dict(d0, idx=np.zeros((bs, 1), np.int32))
    d3["assist"], _ = _layout(d3["idx"], 2, 5, bs)
    d3["y"] = oracle.dispatch_permute(d["x"], d3["assist"], 1, bs)
    assert np.array_equal(_combine(d3, dtype, shared=None), d["x"])


def test_two_copy_experts_scale_ori_x():
    # ids 1 and 2 are copy experts; w = (0.5, 0.25): out = rne(0.75 * ori_x)
    rng = np.random.default_rng(9)
    bs, h = 16, 32
    x = workloads.encode16(rng.standard_normal((bs, h)), "bf16")
    idx = np.tile(np.array([[1, 2]], np.int32), (bs, 1))
    w = np.tile(np.array([[0.5, 0.25]], np.float32), (bs, 1))
    assist, _ = _layout(idx, 1, 3, bs * 2)
    y = np.zeros((bs * 2, h), np.uint16)
    out = oracle.combine_fwd(y, idx, w, assist, num_experts=1, a_capacity=bs * 2, dtype="bf16",
                             copy_expert_num=2, ori_x=x)
    want = workloads.encode16(0.75 * workloads.decode16(x, "bf16").astype(np.float64), "bf16")
    assert np.array_equal(out, want)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("mask_ndim", [0, 2])
def test_combine_bwd(dtype, mask_ndim):
    d = _random_case(dtype, seed=20 + mask_ndim, mask_ndim=mask_ndim, z=0, c=0, q=0)
    bs, k, a_cap = d["bs"], d["k"], d["bs"] * d["k"]
    ge, gw, mag = oracle.combine_bwd(d["g"], d["y"], d["w"], d["assist"], k=k, a_capacity=a_cap,
                                     dtype=dtype, mask=d["mask"])
    g = workloads.decode16(d["g"], dtype).astype(np.float64)
    y = workloads.decode16(d["y"], dtype).astype(np.float64)
    slot = d["assist"][a_cap:].reshape(bs, k)

    # finite differences of L(w) = <g, sum_k w_k y_slot(k)> in float64
    def loss(wv):
        tot = 0.0
        for t in range(bs):
            for kk in range(k):
                if slot[t, kk] >= 0:
                    tot += float(np.dot(g[t], wv[t, kk] * y[slot[t, kk]]))
        return tot
    w64 = d["w"].astype(np.float64)
    for t, kk in [(0, 0), (3, 2), (bs - 1, k - 1), (7, 1)]:
        if slot[t, kk] < 0:
            assert gw[t, kk] == 0
            continue
        step = np.zeros_like(w64)
        step[t, kk] = 1e-3
        fd = (loss(w64 + step) - loss(w64 - step)) / 2e-3
        assert abs(gw[t, kk] - fd) <= 1e-6 * max(1.0, mag[t, kk])
        # grad_expand = w * g rounded once to 16 bits
        got = workloads.decode16(ge[slot[t, kk]], dtype).astype(np.float64)
        ref = w64[t, kk] * g[t]
        tol = np.abs(ref) * (2.0**-8 if dtype == "bf16" else 2.0**-11) * (1 + 2**-20) + 1e-30
        if dtype == "fp16":
            tol = tol + 2.0**-25  # half-ulp of fp16 subnormals
        assert np.all(np.abs(got - ref) <= tol)
    # K = 1, w = 1: grad_expand is grad_out
    idx1 = np.zeros((bs, 1), np.int32)
    a1, _ = _layout(idx1, 1, 1, bs)
    ge1, _, _ = oracle.combine_bwd(d["g"], d["y"][:bs], np.ones((bs, 1), np.float32), a1, k=1,
                                   a_capacity=bs, dtype=dtype)
    assert np.array_equal(ge1, d["g"])
    # masked / slotless pairs: grad_w = 0
    assert np.all(gw[slot < 0] == 0)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_dispatch_bwd(dtype):
    d = _random_case(dtype, seed=31, z=0, c=0, q=0, mask_ndim=2)
    bs, k, a_cap = d["bs"], d["k"], d["bs"] * d["k"]
    gx = oracle.dispatch_bwd(d["y"], d["assist"], bs=bs, k=k, a_capacity=a_cap, dtype=dtype,
                             mask=d["mask"])
    y = workloads.decode16(d["y"], dtype).astype(np.float64)
    slot = d["assist"][a_cap:].reshape(bs, k)
    exact = np.zeros((bs, d["h"]))
    for t in range(bs):
        for kk in range(k):
            if slot[t, kk] >= 0:
                exact[t] += y[slot[t, kk]]
    dist = ulp_dist(gx, workloads.encode16(exact, dtype))
    assert dist.max() <= 1 and (dist == 0).mean() > 0.97
    # K = 1: the gradient returns unchanged
    idx1 = np.zeros((bs, 1), np.int32)
    a1, _ = _layout(idx1, 1, 1, bs)
    assert np.array_equal(oracle.dispatch_bwd(d["y"][:bs], a1, bs=bs, k=1, a_capacity=bs,
                                              dtype=dtype), d["y"][:bs])


def test_chain_runs_on_every_workload_shape():
    for wl in workloads.WORKLOADS:
        small = wl.scaled(bs=48, h=32)
        r = oracle.run_chain(workloads.generate(small))
        assert r["out"].shape == (48, 32)
        if small.backward:
            assert r["grad_x"].shape == (48, 32)


def test_int8_roundtrip_hand_case():
    g = read("combine_int8_roundtrip.txt")
    y = workloads.encode16(np.array(g["y"], np.float32), g["dtype"])
    bs = len(y)
    idx = np.zeros((bs, 1), np.int32)
    assist, _ = _layout(idx, 1, 1, bs)
    out = oracle.combine_fwd(y, idx, np.ones((bs, 1), np.float32), assist, num_experts=1,
                             a_capacity=bs, dtype=g["dtype"], comm_quant_mode=2)
    assert np.array_equal(out, workloads.encode16(np.array(g["out"], np.float32), g["dtype"]))


def test_int8_roundtrip_exact_rows_and_bound():
    rng = np.random.default_rng(41)
    bs, h = 64, 48
    # rows of integers with max |y| = 127: scale 1, the round trip is exact
    yi = rng.integers(-127, 128, (bs, h)).astype(np.float32)
    yi[:, 0] = 127.0
    y_exact = workloads.encode16(yi, "bf16")
    idx = np.zeros((bs, 1), np.int32)
    assist, _ = _layout(idx, 1, 1, bs)
    w1 = np.ones((bs, 1), np.float32)
    kw = dict(num_experts=1, a_capacity=bs, dtype="bf16")
    assert np.array_equal(oracle.combine_fwd(y_exact, idx, w1, assist, comm_quant_mode=2, **kw),
                          y_exact)
    # general rows: within half a quantisation step (plus the bf16 rounding)
    y = workloads.encode16(rng.standard_normal((bs, h)) * 3, "bf16")
    yf = workloads.decode16(y, "bf16").astype(np.float64)
    got = workloads.decode16(oracle.combine_fwd(y, idx, w1, assist, comm_quant_mode=2, **kw),
                             "bf16").astype(np.float64)
    step = np.abs(yf).max(axis=1, keepdims=True) / 127
    assert np.all(np.abs(got - yf) <= step / 2 + np.abs(got) * 2.0**-8 + 1e-30)
    assert not np.array_equal(got, yf)  # the round trip does change some values


def test_int8_roundtrip_leaves_local_terms_alone():
    # copy/const experts and shared_expert_x are not communicated: unchanged by mode 2
    d = _random_case("bf16", k=2, e=2, z=1, c=1, q=1, seed=8)
    bs = d["bs"]
    d["idx"] = np.tile(np.array([[3, 4]], np.int32), (bs, 1))  # copy + const only
    d["assist"], _ = _layout(d["idx"], 2, 5, bs * 2)
    assert np.array_equal(_combine(d, "bf16", comm_quant_mode=2), _combine(d, "bf16"))
