"""Pins of the oracle's dispatch permute and its dynamic int8 quantisation:
hand-computed rows, the bit copy property, and the quantisation error bound."""
import numpy as np
import pytest

import oracle
import workloads
from golden_io import read


def _one_slot_per_token(bs):
    # K = 1, every token routed to expert 0: slot t holds token t
    idx = np.zeros((bs, 1), np.int32)
    _, _, assist, st = oracle.dispatch_layout(idx, 1, 1, bs)
    assert st == 0
    return assist


def test_hand_rows():
    g = read("quant_rows.txt")
    x = np.array(g["x"], np.float32)
    bits = workloads.encode16(x, g["dtype"])
    assist = _one_slot_per_token(len(x))
    q, sc = oracle.dispatch_permute_quant(bits, assist, 1, len(x), g["dtype"])
    assert q.tolist() == g["codes"]
    want = [np.float32(n) / np.float32(d) if n else np.float32(0)
            for n, d in zip(g["scale_num"], g["scale_den"])]
    assert sc.view(np.uint32).tolist() == np.array(want, np.float32).view(np.uint32).tolist()


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_quant_error_bound_and_full_range(dtype):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((300, 96)) * rng.uniform(1e-3, 50, (300, 1))
    x[5] = 0.0
    bits = workloads.encode16(x, dtype)
    xf = workloads.decode16(bits, dtype)
    assist = _one_slot_per_token(300)
    q, sc = oracle.dispatch_permute_quant(bits, assist, 1, 300, dtype)
    for t in range(300):
        amax = np.abs(xf[t]).max()
        if amax == 0:
            assert sc[t] == 0 and not q[t].any()
            continue
        assert np.abs(q[t]).max() == 127
        assert abs(float(sc[t]) - amax / 127.0) <= amax / 127.0 * 2**-23
        err = np.abs(q[t].astype(np.float64) * sc[t] - xf[t])
        assert err.max() <= sc[t] * (0.5 + 2**-16)


def test_permute_is_a_bit_copy_and_quant_replicates():
    wl = workloads.WORKLOADS[4].scaled(bs=64, h=128)
    inp = workloads.generate(wl)
    _, send, assist, st = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                 wl.a_capacity)
    r = int(send[-1])
    ex = oracle.dispatch_permute(inp["x"], assist, wl.k, wl.a_capacity)
    tok = assist[:r] // wl.k
    assert np.array_equal(ex[:r], inp["x"][tok])
    q, sc = oracle.dispatch_permute_quant(inp["x"], assist, wl.k, wl.a_capacity, wl.dtype)
    # every slot of a token carries the token's codes and scale
    q1, sc1 = oracle.dispatch_permute_quant(inp["x"], _one_slot_per_token(wl.bs), 1, wl.bs,
                                            wl.dtype)
    assert np.array_equal(q[:r], q1[tok]) and np.array_equal(sc[:r], sc1[tok])


def test_smooth_scales_pins():
    """Smooth-scaled int8 permute: unit scales reduce to the plain quantisation; a
    power-of-two scale per expert doubles the dequantised row exactly; every slot's
    codes stay within half a step of x * s."""
    wl = workloads.WORKLOADS[4].scaled(bs=96, h=64, zero_expert_num=0, copy_expert_num=0,
                                       const_expert_num=0, num_experts=8)
    inp = workloads.generate(wl)
    _, send, assist, st = oracle.dispatch_layout(inp["topk_idx"], wl.num_experts, wl.n_ids,
                                                 wl.a_capacity)
    r = int(send[-1])
    ones = np.ones((wl.num_experts, wl.h), np.float32)
    q1, s1 = oracle.dispatch_permute_quant(inp["x"], assist, wl.k, wl.a_capacity, wl.dtype)
    q2, s2 = oracle.dispatch_permute_quant_smooth(inp["x"], inp["topk_idx"], ones, assist,
                                                  wl.a_capacity, wl.dtype)
    assert np.array_equal(q1[:r], q2[:r]) and np.array_equal(s1[:r], s2[:r])
    # expert e scaled by 2^e: codes unchanged, scale multiplied by 2^e exactly
    pow2 = np.repeat((2.0 ** np.arange(wl.num_experts, dtype=np.float32))[:, None], wl.h, 1)
    q3, s3 = oracle.dispatch_permute_quant_smooth(inp["x"], inp["topk_idx"], pow2, assist,
                                                  wl.a_capacity, wl.dtype)
    pair = assist[:r]
    e = inp["topk_idx"].reshape(-1)[pair]
    assert np.array_equal(q3[:r], q1[:r])
    assert np.array_equal(s3[:r], (s1[:r] * 2.0 ** e).astype(np.float32))
    # random per-expert scales: the round trip stays within half a step of x * s
    rng = np.random.default_rng(2)
    sm = rng.uniform(0.1, 4.0, (wl.num_experts, wl.h)).astype(np.float32)
    q4, s4 = oracle.dispatch_permute_quant_smooth(inp["x"], inp["topk_idx"], sm, assist,
                                                  wl.a_capacity, wl.dtype)
    xf = workloads.decode16(inp["x"], wl.dtype).astype(np.float64)
    y = xf[pair // wl.k] * sm[e]
    err = np.abs(q4[:r].astype(np.float64) * s4[:r, None] - y)
    assert np.all(err <= s4[:r, None] * (0.5 + 2**-16))
    assert np.all(np.abs(q4[:r]).max(axis=1) == 127)
