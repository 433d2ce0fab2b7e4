"""Pins of the oracle's special-expert backward (copy and const experts): finite
differences of L = sum_t <grad_out[t], out[t]> in float64 for every input, the copy
closed form, and the exchange symmetry of alpha_2 and v."""
import numpy as np
import pytest

import oracle
import workloads


def _case(seed=0, bs=12, h=10, k=3, e=2, z=1, c=2, q=2, dtype="bf16", mask_ndim=0):
    rng = np.random.default_rng(seed)
    n = e + z + c + q
    idx = np.argsort(rng.random((bs, n)), axis=1)[:, :k].astype(np.int32)
    enc = lambda shape: workloads.encode16(rng.standard_normal(shape), dtype)  # noqa: E731
    d = dict(idx=idx, w=rng.uniform(-1, 1, (bs, k)).astype(np.float32), g=enc((bs, h)),
             x=enc((bs, h)), a1=enc((q, h)), a2=enc((q, h)), v=enc((q, h)),
             e=e, z=z, c=c, q=q, bs=bs, h=h, k=k, dtype=dtype, mask=None)
    if mask_ndim == 2:
        d["mask"] = (rng.random((bs, k)) > 0.25).astype(np.uint8)
    return d


def _run(d):
    return oracle.combine_bwd_special(
        d["g"], d["idx"], d["w"], num_experts=d["e"], dtype=d["dtype"], zero_expert_num=d["z"],
        copy_expert_num=d["c"], const_expert_num=d["q"], mask=d["mask"], ori_x=d["x"],
        alpha1=d["a1"], alpha2=d["a2"], const_v=d["v"])


def _loss(d, w, x, a1, a2, v):
    """L = sum_t <g_t, sum over copy/const pairs of w * M> in float64 (no rounding)."""
    f = lambda a: workloads.decode16(a, d["dtype"]).astype(np.float64)  # noqa: E731
    g = f(d["g"])
    tot = 0.0
    lo = d["e"] + d["z"]
    for t in range(d["bs"]):
        for kk in range(d["k"]):
            if d["mask"] is not None and not d["mask"][t, kk]:
                continue
            i = d["idx"][t, kk]
            if i < lo:
                continue
            if i < lo + d["c"]:
                m = x[t]
            else:
                j = i - lo - d["c"]
                m = a1[j] * x[t] + a2[j] * v[j]
            tot += w[t, kk] * float(np.dot(g[t], m))
    return tot


@pytest.mark.parametrize("mask_ndim", [0, 2])
def test_finite_differences(mask_ndim):
    d = _case(seed=3 + mask_ndim, mask_ndim=mask_ndim)
    r = _run(d)
    f = lambda a: workloads.decode16(a, d["dtype"]).astype(np.float64)  # noqa: E731
    base = dict(w=d["w"].astype(np.float64), x=f(d["x"]), a1=f(d["a1"]), a2=f(d["a2"]),
                v=f(d["v"]))
    eps = 1e-3

    def fd(name, index):
        up = {k: v.copy() for k, v in base.items()}
        dn = {k: v.copy() for k, v in base.items()}
        up[name][index] += eps
        dn[name][index] -= eps
        return (_loss(d, **up) - _loss(d, **dn)) / (2 * eps)

    lo = d["e"] + d["z"]
    special = (d["idx"] >= lo)
    if d["mask"] is not None:
        special &= d["mask"].astype(bool)
    for t, kk in zip(*np.nonzero(special)):
        assert abs(r["grad_w"][t, kk] - fd("w", (t, kk))) <= 1e-6 * max(1.0, r["abs_sum"][t, kk])
    assert np.all(r["grad_w"][~special] == 0)
    for name, key, absk in (("a1", "grad_alpha1", "abs_alpha1"), ("a2", "grad_alpha2", "abs_alpha2"),
                            ("v", "grad_v", "abs_v")):
        for j in range(d["q"]):
            for col in (0, 3, d["h"] - 1):
                assert abs(r[key][j, col] - fd(name, (j, col))) <= \
                    1e-5 * max(1.0, r[absk][j, col])
    gx = workloads.decode16(r["grad_ori_x"], d["dtype"]).astype(np.float64)
    for t in (0, 5, d["bs"] - 1):
        for col in (0, 7):
            want = fd("x", (t, col))
            assert abs(gx[t, col] - want) <= abs(want) * 2.0**-7 + 1e-6


def test_copy_closed_form_and_symmetry():
    # one copy expert, weight 1: grad_ori_x = grad_out exactly, grad_w = <g, ori_x>
    d = _case(seed=9, k=1, e=1, z=0, c=1, q=0)
    d["idx"][:] = 1
    d["w"][:] = 1.0
    r = _run(d)
    assert np.array_equal(r["grad_ori_x"], d["g"])
    f = lambda a: workloads.decode16(a, "bf16").astype(np.float64)  # noqa: E731
    assert np.allclose(r["grad_w"][:, 0], np.sum(f(d["g"]) * f(d["x"]), axis=1), rtol=1e-6)
    # const expert with alpha_2 == v: grad_alpha2 and grad_v coincide
    d = _case(seed=10, k=2, e=1, z=0, c=0, q=1)
    d["idx"][:, 0] = 0
    d["idx"][:, 1] = 1
    d["a2"] = d["v"].copy()
    r = _run(d)
    assert np.array_equal(r["grad_alpha2"], r["grad_v"])
    # alpha_1 = 1, alpha_2 = 0 makes the const expert a copy expert
    d2 = _case(seed=11, k=1, e=1, z=0, c=1, q=1)
    d2["idx"][:] = 2  # const expert 0
    d2["a1"] = workloads.encode16(np.ones((1, d2["h"])), "bf16")
    d2["a2"] = workloads.encode16(np.zeros((1, d2["h"])), "bf16")
    rc = _run(d2)
    d2c = dict(d2, idx=np.full_like(d2["idx"], 1))  # the copy expert
    rcopy = _run(d2c)
    assert np.array_equal(rc["grad_ori_x"], rcopy["grad_ori_x"])
    assert np.array_equal(rc["grad_w"], rcopy["grad_w"])
