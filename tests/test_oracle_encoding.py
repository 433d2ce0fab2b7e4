"""Pins of the oracle's 16-bit float encodings against independent library
conversions (numpy float16, torch bfloat16): exhaustive for decoding, random
patterns plus every rounding tie for encoding."""
import numpy as np
import pytest
import torch

import oracle


def _torch_bf16(f32):
    return torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_decode_exhaustive_fp16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode16_array(bits, "fp16")
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_decode_exhaustive_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode16_array(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _probe_values(dtype):
    """Random fp32 patterns plus, for every pair of neighbouring 16-bit values,
    their midpoint (a tie) and the fp32 values just around it."""
    rng = np.random.default_rng(7)
    rnd = rng.integers(0, 2**32, 400_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    lo = np.arange(0, 0x7C00 if dtype == "fp16" else 0x7F80, dtype=np.uint32).astype(np.uint16)
    f_lo = oracle.decode16_array(lo, dtype).astype(np.float64)
    f_hi = oracle.decode16_array((lo + 1).astype(np.uint16), dtype).astype(np.float64)
    mid = ((f_lo + f_hi) / 2).astype(np.float32)  # exact: fp32 holds every midpoint
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(-np.inf))
    v = np.concatenate([rnd, mid, up, dn, -mid, -up, -dn,
                        np.array([0.0, -0.0, 65504, 65519.99, 65520, 1e-8, -1e-8,
                                  np.inf, -np.inf], np.float32)])
    return v[~np.isnan(v)]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_encode_rne_matches_library(dtype):
    v = _probe_values(dtype)
    got = oracle.encode16_array(v, dtype)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16) if dtype == "fp16" else _torch_bf16(v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (dtype, v[bad[:5]], got[bad[:5]], ref[bad[:5]])
