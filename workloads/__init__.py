"""Seeded synthetic inputs for MoE token dispatch and combine.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It holds only random draws, the 16-bit encoding of those draws, and the
untimed "expert" stand-ins that sit between dispatch and combine. None of the
dispatch/combine arithmetic lives here.

The five workloads follow the shapes the problem is posed on: the Ascend
``low_latency_combine`` page (Parameters table: topk_idx (BS, K) int32, topk_weights
(BS, K) fp32, x (A, H) bf16/fp16, x_active_mask (BS,) or (BS, K), shared_expert_x
(BS, H), ori_x and the const-expert tensors (Q, H)) and the MoE-layer shapes named
by the Megatron-LM "Add performance test for MoE layer" page (DeepSeek-V3 and
Mixtral-8x7B proxies).

Recipe (all draws from one ``numpy.random.PCG64(seed)`` stream, in this order):
  1. routing: uniform distinct ids over the N = E+Z+C+Q id range (a random
     permutation per token, first K kept), or Zipf(s) popularity
     p_i ~ (i+1)^-s drawn without replacement (Gumbel top-K, which samples the
     same law as sequential weighted draws);
  2. weight logits ~ N(0,1) (BS, K) in float64 -> softmax or normalised sigmoid
     -> float32;
  3. x ~ N(0,1) (BS, H), float64 -> float32 -> 16-bit (round to nearest even);
  4. optional 2-D mask: (token, k) pair inactive when U(0,1) < p_false;
  5. optional shared_expert_x ~ N(0,1) (BS, H);
  6. optional const-expert alpha_1, alpha_2, v ~ U(-1,1) (Q, H);
  7. optional per-expanded-row expert factor 1+eps, eps ~ U(-0.1, 0.1), float32;
  8. optional grad_out ~ N(0,1) (BS, H).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np

DTYPE_CODES = {"bf16": 0, "fp16": 1}


@dataclass(frozen=True)
class Workload:
    name: str
    bs: int
    h: int
    k: int
    num_experts: int
    zero_expert_num: int = 0
    copy_expert_num: int = 0
    const_expert_num: int = 0
    dtype: str = "bf16"
    routing: str = "uniform"          # "uniform" | "zipf"
    zipf_s: float = 1.1
    weights: str = "softmax"          # "softmax" | "sigmoid_norm"
    expert: str = "identity"          # "identity" | "eps" | "dequant"
    shared: bool = False
    mask_ndim: int = 0                # 0 none, 1 (BS,), 2 (BS, K)
    mask_false_p: float = 0.0
    quant_mode: int = 0               # 0 none, 2 dynamic int8 per row
    smooth: bool = False              # int8 of x * smooth_scales[e] (needs quant_mode 2)
    backward: bool = True
    seed: int = 1
    a_capacity_override: int = 0

    @property
    def n_ids(self) -> int:
        return (self.num_experts + self.zero_expert_num + self.copy_expert_num
                + self.const_expert_num)

    @property
    def a_capacity(self) -> int:
        return self.a_capacity_override or self.bs * self.k

    @property
    def elem_bytes(self) -> int:
        return 2

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads, in order: a tiny forward-only case, the 8192-token
# H=1536 case the headline throughput is quoted on, a DeepSeek-V3-shaped case,
# a Mixtral-shaped case, and a special-expert + int8 forward case.
WORKLOADS = [
    Workload("tiny_bs128_h1536_k8_e64", bs=128, h=1536, k=8, num_experts=64,
             backward=False, seed=1),
    Workload("uniform_bs8192_h1536_k8_e64", bs=8192, h=1536, k=8, num_experts=64,
             expert="eps", backward=True, seed=2),
    Workload("dsv3_bs4096_h7168_k8_e256", bs=4096, h=7168, k=8, num_experts=256,
             routing="zipf", zipf_s=1.1, weights="sigmoid_norm", shared=True,
             backward=True, seed=3),
    Workload("mixtral_bs16384_h4096_k2_e8", bs=16384, h=4096, k=2, num_experts=8,
             dtype="fp16", mask_ndim=2, mask_false_p=0.1, backward=True, seed=4),
    Workload("special_int8_bs8192_h2048_k8_n70", bs=8192, h=2048, k=8, num_experts=64,
             zero_expert_num=2, copy_expert_num=2, const_expert_num=2,
             expert="dequant", quant_mode=2, backward=False, seed=5),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def encode16(a: np.ndarray, dtype: str) -> np.ndarray:
    """float32/float64 array -> uint16 bit patterns of bf16/fp16, round to nearest even."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    return t.to(tdt).view(torch.int16).numpy().view(np.uint16)


def decode16(bits: np.ndarray, dtype: str) -> np.ndarray:
    """uint16 bit patterns of bf16/fp16 -> float32 (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits.view(np.float16).astype(np.float32)


def _routing(rng: np.random.Generator, wl: Workload) -> np.ndarray:
    n = wl.n_ids
    if wl.k > n:
        raise ValueError("K larger than the id range")
    if wl.routing == "uniform":
        keys = rng.random((wl.bs, n))
    elif wl.routing == "zipf":
        logp = -wl.zipf_s * np.log(np.arange(1, n + 1, dtype=np.float64))
        u = rng.random((wl.bs, n))
        u = np.clip(u, 1e-300, 1.0)
        keys = logp[None, :] - np.log(-np.log(u))
        keys = -keys  # argsort ascending -> largest key first
    else:
        raise ValueError(wl.routing)
    order = np.argsort(keys, axis=1, kind="stable")[:, : wl.k]
    return np.ascontiguousarray(order.astype(np.int32))


def _weights(rng: np.random.Generator, wl: Workload) -> np.ndarray:
    logits = rng.standard_normal((wl.bs, wl.k))
    if wl.weights == "softmax":
        z = np.exp(logits - logits.max(axis=1, keepdims=True))
        w = z / z.sum(axis=1, keepdims=True)
    elif wl.weights == "sigmoid_norm":
        s = 1.0 / (1.0 + np.exp(-logits))
        w = s / s.sum(axis=1, keepdims=True)
    else:
        raise ValueError(wl.weights)
    return np.ascontiguousarray(w.astype(np.float32))


def generate(wl: Workload, seed: int | None = None) -> dict:
    """Draw one workload's inputs. All 16-bit tensors are uint16 bit patterns."""
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    out: dict = {"workload": wl}
    out["topk_idx"] = _routing(rng, wl)
    out["topk_weights"] = _weights(rng, wl)
    out["x"] = encode16(rng.standard_normal((wl.bs, wl.h)), wl.dtype)
    out["mask"] = None
    if wl.mask_ndim == 2:
        out["mask"] = (rng.random((wl.bs, wl.k)) >= wl.mask_false_p).astype(np.uint8)
    elif wl.mask_ndim == 1:
        out["mask"] = (rng.random(wl.bs) >= wl.mask_false_p).astype(np.uint8)
    out["shared"] = (encode16(rng.standard_normal((wl.bs, wl.h)), wl.dtype)
                     if wl.shared else None)
    q = wl.const_expert_num
    if q:
        out["alpha1"] = encode16(rng.uniform(-1.0, 1.0, (q, wl.h)), wl.dtype)
        out["alpha2"] = encode16(rng.uniform(-1.0, 1.0, (q, wl.h)), wl.dtype)
        out["v"] = encode16(rng.uniform(-1.0, 1.0, (q, wl.h)), wl.dtype)
    else:
        out["alpha1"] = out["alpha2"] = out["v"] = None
    # ori_x is the token data before the experts, i.e. the same tensor as x.
    out["ori_x"] = out["x"] if (wl.copy_expert_num or q) else None
    out["expert_factor"] = None
    if wl.expert == "eps":
        eps = rng.uniform(-0.1, 0.1, wl.a_capacity)
        out["expert_factor"] = (1.0 + eps).astype(np.float32)
    out["grad_out"] = (encode16(rng.standard_normal((wl.bs, wl.h)), wl.dtype)
                       if wl.backward else None)
    out["smooth"] = smooth_scales(wl, seed) if wl.smooth else None
    return out


def smooth_scales(wl: Workload, seed: int | None = None) -> np.ndarray:
    """Per-expert, per-channel smooth-quant factors (E, H) fp32, standard normal
    like the graph-mode dispatch example's scales; drawn from their own stream so
    that generate() is unchanged."""
    rng = np.random.Generator(np.random.PCG64((wl.seed if seed is None else seed) + 7919))
    return np.ascontiguousarray(
        rng.standard_normal((wl.num_experts, wl.h)).astype(np.float32))


# ---------------------------------------------------------------------------
# Untimed expert stand-ins (the experts' FFN is outside the dispatch/combine
# path; these give combine non-trivial inputs of the right shape).
# ---------------------------------------------------------------------------

def expert_forward(inputs: dict, expand_x: np.ndarray,
                   dynamic_scales: np.ndarray | None = None) -> np.ndarray:
    """Expert outputs Y (A, H) as uint16 bit patterns from dispatch's expanded rows.

    identity: Y = expand_x.  eps: Y[s] = round16(float(expand_x[s]) * f[s]).
    dequant:  Y[s] = round16(float(q[s]) * scale[s])  (int8 rows with per-row scale).
    """
    wl: Workload = inputs["workload"]
    if wl.expert == "identity":
        return np.array(expand_x, dtype=np.uint16, copy=True)
    if wl.expert == "eps":
        f = inputs["expert_factor"]
        y = decode16(expand_x, wl.dtype) * f[:, None]
        return encode16(y, wl.dtype)
    if wl.expert == "dequant":
        assert dynamic_scales is not None
        y = expand_x.astype(np.float32) * dynamic_scales.astype(np.float32)[:, None]
        return encode16(y, wl.dtype)
    raise ValueError(wl.expert)


def expert_backward(inputs: dict, grad_y: np.ndarray) -> np.ndarray:
    """Gradient w.r.t. the experts' inputs from the gradient w.r.t. their outputs."""
    wl: Workload = inputs["workload"]
    if wl.expert == "eps":
        g = decode16(grad_y, wl.dtype) * inputs["expert_factor"][:, None]
        return encode16(g, wl.dtype)
    return np.array(grad_y, dtype=np.uint16, copy=True)
