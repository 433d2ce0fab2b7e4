"""Runs the whole path through the C ABI on the GPU and the CPU oracle on the same
seeded inputs, stage by stage. Every stage on both sides gets the same inputs: the
expert stand-ins between dispatch and combine run once on the host, on the
oracle's (already compared) dispatch output."""
from __future__ import annotations

import numpy as np
import torch

import combine_moe_dispatch_04_b200 as moe
import oracle
import workloads

# Tolerances: 16-bit outputs within one ulp; grad_w within 1e-5 relative to
# max(|grad_w|, sum_h |grad_out * expand_x|).
ULP_TOL = 1
GRAD_W_RTOL = 1e-5


def shape_of(wl: workloads.Workload) -> moe.Shape:
    return moe.Shape(bs=wl.bs, k=wl.k, h=wl.h, num_experts=wl.num_experts,
                     zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
                     const_expert_num=wl.const_expert_num, a_capacity=wl.a_capacity,
                     dtype=workloads.DTYPE_CODES[wl.dtype], mask_ndim=wl.mask_ndim)


def dev(a, dtype16: str | None = None):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).cuda()
        return t.view(torch.bfloat16 if dtype16 == "bf16" else torch.float16)
    return torch.from_numpy(a).cuda()


def host(t) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def ulp_dist(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordered(a) - ordered(b))


class Mismatch(AssertionError):
    pass


def _eq(name, got, want):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise Mismatch(f"{name}: {len(bad)} mismatches, first at {bad[:3].tolist()}")


def _ulp(name, got, want, rows=None):
    if rows is not None:
        got, want = got[rows], want[rows]
    d = ulp_dist(got, want)
    if d.size and d.max() > ULP_TOL:
        bad = np.argwhere(d > ULP_TOL)
        raise Mismatch(f"{name}: {len(bad)} elements beyond {ULP_TOL} ulp, first {bad[:3].tolist()}")
    return float((d == 0).mean()) if d.size else 1.0


def run_compare(inputs: dict, *, twice: bool = False) -> dict:
    """GPU vs oracle on one workload. Raises Mismatch on any disagreement.
    Returns a small report (exact-match fractions, max grad_w error)."""
    wl = inputs["workload"]
    dt = wl.dtype
    sh = shape_of(wl)
    rep: dict = {}
    ref = oracle.run_chain(inputs)
    r = int(ref["send"][-1])

    idx_d = dev(inputs["topk_idx"])
    mask_d = dev(inputs["mask"])
    lay = moe.dispatch_layout(sh, idx_d, mask_d)
    torch.cuda.synchronize()
    _eq("expert_token_nums", host(lay.expert_token_nums), ref["counts"])
    _eq("ep_send_counts", host(lay.ep_send_counts), ref["send"])
    _eq("assist_info", host(lay.assist_info), ref["assist"])
    _eq("dev_status", host(lay.dev_status).astype(np.int64) & 3, np.array([ref["status"]]))

    x_d = dev(inputs["x"], dt)
    if wl.quant_mode == 2:
        q_d, sc_d = moe.dispatch_permute(sh, x_d, lay, 2)
        torch.cuda.synchronize()
        _eq("int8 codes", host(q_d)[:r], ref["expand_q"][:r])
        _eq("dynamic_scales", host(sc_d)[:r].view(np.uint32), ref["scales"][:r].view(np.uint32))
    else:
        ex_d, _ = moe.dispatch_permute(sh, x_d, lay, 0)
        torch.cuda.synchronize()
        _eq("expand_x", host(ex_d)[:r], ref["expand_x"][:r])

    y_d = dev(ref["y"], dt)
    w_d = dev(inputs["topk_weights"])
    out_d = moe.combine_fwd(sh, y_d, idx_d, w_d, lay, x_active_mask=mask_d,
                            shared_expert_x=dev(inputs["shared"], dt),
                            ori_x=dev(inputs["ori_x"], dt), const_alpha_1=dev(inputs["alpha1"], dt),
                            const_alpha_2=dev(inputs["alpha2"], dt), const_v=dev(inputs["v"], dt))
    torch.cuda.synchronize()
    out = host(out_d)
    rep["combine_exact"] = _ulp("combine out", out, ref["out"])

    if wl.backward:
        g_d = dev(inputs["grad_out"], dt)
        ge_d, gw_d = moe.combine_bwd(sh, g_d, y_d, w_d, lay, x_active_mask=mask_d)
        torch.cuda.synchronize()
        ge, gw = host(ge_d), host(gw_d)
        rep["grad_expand_exact"] = _ulp("grad_expand", ge[:r], ref["grad_expand"][:r])
        err = np.abs(gw.astype(np.float64) - ref["grad_w"].astype(np.float64))
        bound = GRAD_W_RTOL * np.maximum(np.abs(ref["grad_w"].astype(np.float64)), ref["abs_sum"])
        if np.any(err > bound):
            bad = np.argwhere(err > bound)
            raise Mismatch(f"grad_w: {len(bad)} beyond tolerance, first {bad[:3].tolist()}")
        rep["grad_w_max_rel"] = float(np.max(err / np.maximum(bound / GRAD_W_RTOL, 1e-30))) \
            if err.size else 0.0
        gi_d = dev(ref["grad_in"], dt)
        gx_d = moe.dispatch_bwd(sh, gi_d, lay, x_active_mask=mask_d)
        torch.cuda.synchronize()
        rep["grad_x_exact"] = _ulp("grad_x", host(gx_d), ref["grad_x"])

    if twice:  # determinism: a second run gives the same bits
        lay2 = moe.dispatch_layout(sh, idx_d, mask_d)
        out2 = moe.combine_fwd(sh, y_d, idx_d, w_d, lay2, x_active_mask=mask_d,
                               shared_expert_x=dev(inputs["shared"], dt),
                               ori_x=dev(inputs["ori_x"], dt),
                               const_alpha_1=dev(inputs["alpha1"], dt),
                               const_alpha_2=dev(inputs["alpha2"], dt),
                               const_v=dev(inputs["v"], dt))
        torch.cuda.synchronize()
        _eq("assist (rerun)", host(lay2.assist_info), host(lay.assist_info))
        _eq("combine out (rerun)", host(out2), out)
        if wl.backward:
            ge2, gw2 = moe.combine_bwd(sh, g_d, y_d, w_d, lay2, x_active_mask=mask_d)
            torch.cuda.synchronize()
            _eq("grad_w (rerun)", host(gw2).view(np.uint32), gw.view(np.uint32))
    return rep
