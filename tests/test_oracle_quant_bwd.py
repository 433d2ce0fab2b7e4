"""Pins of the oracle's backward of the int8 round-trip combine (comm_quant_mode 2):
the straight-through reading of the round trip (grad_expand as without
quantisation), grad_w against values fixed by the already-pinned int8 dispatch
quantisation, rows the round trip leaves unchanged, a finite difference of the
pinned forward, and the masked / slotless pairs."""
import numpy as np
import pytest

import oracle
import workloads


def _layout(idx, e, n, a_cap, mask=None):
    _, send, assist, st = oracle.dispatch_layout(idx, e, n, a_cap, mask)
    assert st == 0
    return assist


def _case(dtype, bs=30, h=40, k=3, e=5, seed=0, mask=False):
    rng = np.random.default_rng(seed)
    idx = np.argsort(rng.random((bs, e)), axis=1)[:, :k].astype(np.int32)
    w = rng.uniform(-1, 1, (bs, k)).astype(np.float32)
    m = (rng.random((bs, k)) > 0.25).astype(np.uint8) if mask else None
    a_cap = bs * k
    assist = _layout(idx, e, e, a_cap, m)
    # rows with a few large values, so the round trip moves most of them a lot
    y = rng.standard_normal((a_cap, h)) * rng.uniform(0.01, 5, (a_cap, 1))
    y[:, 0] *= 40
    g = workloads.encode16(rng.standard_normal((bs, h)), dtype)
    return dict(idx=idx, w=w, mask=m, assist=assist, y=workloads.encode16(y, dtype), g=g,
                bs=bs, h=h, k=k, a_cap=a_cap, e=e)


def _bwd(d, dtype, mode):
    return oracle.combine_bwd(d["g"], d["y"], d["w"], d["assist"], k=d["k"],
                              a_capacity=d["a_cap"], dtype=dtype, mask=d["mask"],
                              comm_quant_mode=mode)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("mask", [False, True])
def test_grad_w_is_the_dot_with_the_dispatch_quantisation(dtype, mask):
    """grad_w = <g, q * scale> with (q, scale) the per-row codes and scale of the
    int8 dispatch quantisation (pinned on its own), summed here by numpy in float64;
    grad_expand is the unquantised backward's, bit for bit."""
    d = _case(dtype, seed=3 + mask, mask=mask)
    ge, gw, mag = _bwd(d, dtype, 2)
    ge0, gw0, _ = _bwd(d, dtype, 0)
    assert np.array_equal(ge, ge0)  # the round trip is passed straight through
    # the rows through the pinned dispatch quantisation: K = 1, row s -> slot s
    a = d["a_cap"]
    ident = _layout(np.zeros((a, 1), np.int32), 1, 1, a)
    q, sc = oracle.dispatch_permute_quant(d["y"], ident, 1, a, dtype)
    deq = (q.astype(np.float32) * sc[:, None]).astype(np.float64)  # the fp32 value q * scale
    g = workloads.decode16(d["g"], dtype).astype(np.float64)
    slot = d["assist"][a:].reshape(d["bs"], d["k"])
    for t in range(d["bs"]):
        for kk in range(d["k"]):
            s = slot[t, kk]
            active = d["mask"] is None or d["mask"][t, kk]
            if s < 0 or not active:
                assert gw[t, kk] == 0 and mag[t, kk] == 0
                continue
            want = float(np.dot(g[t], deq[s]))
            assert abs(float(gw[t, kk]) - want) <= 1e-12 * mag[t, kk] + abs(want) * 2.0**-24
            assert mag[t, kk] == pytest.approx(float(np.abs(g[t] * deq[s]).sum()), rel=1e-12)
    # the round trip changes the dot: the rows were chosen so it moves values a lot
    assert np.abs(gw - gw0).max() > 1e-3


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_rows_the_round_trip_keeps(dtype):
    """Integer rows with max |y| = 127 times a power of two come back unchanged from
    the round trip, so both backwards agree bit for bit."""
    rng = np.random.default_rng(11)
    d = _case(dtype, seed=5)
    yi = rng.integers(-127, 128, (d["a_cap"], d["h"])).astype(np.float64)
    yi[:, 0] = 127
    yi *= 2.0 ** rng.integers(-8, 2, (d["a_cap"], 1))
    d["y"] = workloads.encode16(yi, dtype)
    ge, gw, mag = _bwd(d, dtype, 2)
    ge0, gw0, mag0 = _bwd(d, dtype, 0)
    assert np.array_equal(ge, ge0)
    assert np.array_equal(gw.view(np.uint32), gw0.view(np.uint32))
    assert np.array_equal(mag, mag0)


def test_finite_difference_of_the_forward():
    """grad_w against central differences of L(w) = <g, out(w)> in float64, out the
    oracle's (pinned) forward with comm_quant_mode 2, K = 1: out is rne16(w * D(y)),
    so a difference of L over 2 delta carries at most sum |g| * half an ulp of out
    per evaluation, divided by delta."""
    rng = np.random.default_rng(21)
    bs, h = 12, 64
    y = rng.standard_normal((bs, h)) * rng.uniform(0.1, 3, (bs, 1))
    y[:, 0] *= 30
    y16 = workloads.encode16(y, "bf16")
    idx = np.zeros((bs, 1), np.int32)
    assist = _layout(idx, 1, 1, bs)
    g16 = workloads.encode16(rng.standard_normal((bs, h)), "bf16")
    g = workloads.decode16(g16, "bf16").astype(np.float64)
    w0 = rng.uniform(0.5, 1.5, (bs, 1)).astype(np.float32)
    _, gw, _ = oracle.combine_bwd(g16, y16, w0, assist, k=1, a_capacity=bs, dtype="bf16",
                                  comm_quant_mode=2)

    def loss(w):
        out = oracle.combine_fwd(y16, idx, w.astype(np.float32), assist, num_experts=1,
                                 a_capacity=bs, dtype="bf16", comm_quant_mode=2)
        o = workloads.decode16(out, "bf16").astype(np.float64)
        return (g * o).sum(axis=1), o

    delta = 0.25
    lp, op = loss(w0 + delta)
    lm, om = loss(w0 - delta)
    fd = (lp - lm) / (2 * delta)
    bound = ((np.abs(g) * np.abs(op)).sum(axis=1) + (np.abs(g) * np.abs(om)).sum(axis=1)) \
        * 2.0**-9 / (2 * delta)
    assert np.all(np.abs(fd - gw[:, 0].astype(np.float64)) <= bound + 1e-6)
    # the unquantised gradient misses by more than that bound on these rows
    _, gw0, _ = oracle.combine_bwd(g16, y16, w0, assist, k=1, a_capacity=bs, dtype="bf16")
    assert np.any(np.abs(fd - gw0[:, 0].astype(np.float64)) > bound + 1e-6)
