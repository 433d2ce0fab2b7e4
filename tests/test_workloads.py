"""The seeded input generators: determinism, shapes and the stated distributions."""
import numpy as np
import pytest

import workloads


@pytest.mark.parametrize("wl", workloads.WORKLOADS, ids=lambda w: w.name)
def test_shapes_and_determinism(wl):
    small = wl.scaled(bs=256, h=64)
    a, b = workloads.generate(small), workloads.generate(small)
    for key in ("topk_idx", "topk_weights", "x"):
        assert np.array_equal(a[key], b[key])
    idx = a["topk_idx"]
    assert idx.shape == (256, wl.k) and idx.dtype == np.int32
    assert idx.min() >= 0 and idx.max() < wl.n_ids
    assert all(len(set(r)) == wl.k for r in idx.tolist())  # distinct ids per row
    w = a["topk_weights"]
    assert w.dtype == np.float32 and np.allclose(w.sum(1), 1.0, atol=1e-5) and (w > 0).all()
    assert a["x"].shape == (256, 64) and a["x"].dtype == np.uint16
    assert (a["grad_out"] is not None) == wl.backward
    assert (a["shared"] is not None) == wl.shared
    if wl.const_expert_num:
        assert a["alpha1"].shape == (wl.const_expert_num, 64)
        assert a["ori_x"] is a["x"]


def test_zipf_is_skewed_and_mask_rate():
    dsv3 = workloads.WORKLOADS[2].scaled(bs=2048, h=8)
    idx = workloads.generate(dsv3)["topk_idx"]
    cnt = np.bincount(idx.ravel(), minlength=dsv3.num_experts)
    assert cnt[0] == cnt.max() and cnt[0] > 4 * np.median(cnt)
    mix = workloads.WORKLOADS[3].scaled(bs=8192, h=8)
    m = workloads.generate(mix)["mask"]
    assert m.shape == (8192, 2) and abs((m == 0).mean() - 0.1) < 0.01


def test_encode_decode_roundtrip():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(1000).astype(np.float32)
    for dt in ("bf16", "fp16"):
        bits = workloads.encode16(v, dt)
        assert np.array_equal(workloads.encode16(workloads.decode16(bits, dt), dt), bits)
