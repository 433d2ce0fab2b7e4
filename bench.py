"""Benchmark of the MoE dispatch + combine forward + backward path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  moe_dispatch_layout -> moe_dispatch_permute -> moe_combine_fwd -> moe_combine_bwd
  -> moe_dispatch_bwd
(forward-only workloads stop after moe_combine_fwd). The experts between dispatch and
combine are outside the path: their outputs (and input gradients) are computed once,
untimed, and stay resident in HBM like every other input.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on the host cores

Prints one JSON line (rank 0): the headline workload (the largest single-GPU one,
DeepSeek-V3-shaped, by default) with its roofline, end-to-end and CPU-baseline
figures, plus a per-workload block timing all five workloads in the same process.

Statistics follow the Megatron-LM MoE performance test's method: warm-up steps, then
timed steps; the 3 slowest are dropped and the rest give the mean and standard
deviation; a run is accepted when std/mean <= 2 %, and is repeated up to 5 times
otherwise (the run with the smallest std/mean is kept and marked not accepted).

Multi-GPU runs are independent replicas (one process per GPU, launched with
torch.distributed.run). The process group is gloo on the host: only the barrier and
the max over ranks of the timed duration cross ranks, and no collective touches
device memory.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime as _dt
import hashlib
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "dispatch+combine fwd+bwd tokens/s and achieved HBM GB/s (% of 8 TB/s), 1×B200"
# The largest configuration that fits one GPU: 2644 MB of algorithmic bytes per step.
DEFAULT_WORKLOAD = "dsv3_bs4096_h7168_k8_e256"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
KERNELS = ("layout", "permute", "combine_fwd", "combine_bwd", "combine_bwd_special",
           "dispatch_bwd")
DOM_EVERY = 4
FUSED_DISPATCH_MAX_TOKENS = 1024  # moe_dispatch is one launch up to this batch
DROP_TOP = 3          # slowest steps dropped before the mean and std
ACCEPT_CV = 0.02      # std / mean at or below which a run is accepted
MAX_RUNS = 5          # runs of one workload before the best one is kept
TARGET_FRAC_OF_8TBS = 0.70


# ---------------------------------------------------------------------------
# Algorithmic bytes per launch (each tensor counted once).

def byte_model(wl: workloads.Workload, r: int, ori_tokens: int) -> dict:
    bs, k, h, e = wl.bs, wl.k, wl.h, wl.elem_bytes
    row, pairs = h * e, bs * k
    mask = 0 if wl.mask_ndim == 0 else (bs if wl.mask_ndim == 1 else pairs)
    slot_map = 4 * pairs
    m = {}
    m["layout"] = 4 * pairs + mask + 4 * (wl.a_capacity + pairs) + 4 * (2 * wl.num_experts + 1)
    if wl.quant_mode == 2 and wl.smooth:
        # x once, the smooth factors once, per slot its pair, id, int8 row and scale
        m["permute"] = bs * row + 4 * wl.num_experts * h + 8 * r + r * h + 4 * r
    elif wl.quant_mode == 2:
        m["permute"] = bs * row + slot_map + r * h + 4 * r
    else:
        m["permute"] = bs * row + slot_map + r * row
    special = wl.zero_expert_num + wl.copy_expert_num + wl.const_expert_num
    m["combine_fwd"] = (r * row + 4 * pairs + slot_map + (4 * pairs if special else 0) + mask
                        + (bs * row if wl.shared else 0) + ori_tokens * row
                        + 3 * wl.const_expert_num * row + bs * row)
    if wl.backward:
        m["combine_bwd"] = bs * row + 2 * r * row + 4 * pairs + slot_map + 4 * pairs + mask
        if wl.copy_expert_num + wl.const_expert_num:
            # grad_out and ori_x of the tokens with a copy/const pair, grad_ori_x of
            # every token, ids and weights, the const rows and their gradients
            m["combine_bwd_special"] = (2 * ori_tokens * row + bs * row + 8 * pairs + mask
                                        + 3 * wl.const_expert_num * row
                                        + 3 * wl.const_expert_num * h * 4)
        m["dispatch_bwd"] = r * row + bs * row + slot_map + mask
    return m


# ---------------------------------------------------------------------------
# Replicas: only the timing is reduced across ranks (max), never data. The group is
# gloo, so the reduction runs on the host.

def reduce_max(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    del device  # the reduction runs on a host tensor (gloo)
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(tokens_per_rank_step: int, steps: int, world: int,
                         max_total_ms: float) -> float:
    """Tokens of all replicas divided by the slowest replica's time."""
    return tokens_per_rank_step * steps * world / (max_total_ms * 1e-3)


def trimmed_stats(step_ms: list, drop: int = DROP_TOP) -> dict:
    """Mean and population std of the step times without the `drop` slowest (all of
    them when there are too few steps to drop any)."""
    kept = sorted(step_ms)[:-drop] if len(step_ms) > 2 * drop else list(step_ms)
    mean = statistics.fmean(kept)
    std = statistics.pstdev(kept) if len(kept) > 1 else 0.0
    return {"mean": mean, "std": std, "cv": std / mean if mean > 0 else 0.0,
            "kept": len(kept), "dropped": len(step_ms) - len(kept),
            "plain_mean": statistics.fmean(step_ms), "median": statistics.median(step_ms),
            "max": max(step_ms), "min": min(step_ms)}


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.

class ClockSampler:
    FIELDS = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = (uuid or "").lower()
        self.proc = None
        self.path = None

    def start(self):
        exe = shutil.which("nvidia-smi")
        if exe is None:
            return
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen([exe, f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", "20"],
                                     stdout=self.f, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self, t0: float, t1: float) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            p = [c.strip() for c in line.split(",")]
            if len(p) < 10:
                continue
            if self.uuid and self.uuid not in p[1].lower():
                continue
            try:
                ts = _dt.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(p[2]), float(p[3]), p[6:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        self.proc = None
        inside = [r for r in rows if t0 - 0.02 <= r[0] <= t1 + 0.02]
        window = "timed region"
        if not inside:  # timed region shorter than the sampling period
            inside = [r for r in rows if r[0] <= t1 + 0.1][-3:]
            window = "samples nearest the timed region"
        if not inside:
            return None
        reasons = sorted({self.REASONS[i] for r in inside for i, v in enumerate(r[3])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside), "window": window}


# ---------------------------------------------------------------------------

def layout_launches(bs: int, num_experts: int, k: int) -> int:
    """Launches of moe_dispatch_layout: one thread-block cluster for BS <= 16384 when
    its lane masks and pair lists fit in shared memory, else count, column scan and
    scatter."""
    nt = (256 if bs <= 256 and num_experts <= 256
          else 512 if bs <= 8192 and num_experts <= 512 else 1024)
    stride = num_experts | 1
    smem = (nt // 32) * stride * 8 + num_experts * 12 + nt * k * 4
    return 1 if bs <= 16384 and smem <= 210 * 1024 else 3


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {"layout": "layout.cu", "dispatch": "layout.cu", "permute": "permute.cu",
                  "combine_fwd": "combine.cu", "combine_bwd_special": "special_bwd.cu",
                  "combine_bwd": "combine_bwd.cu", "dispatch_bwd": "combine.cu"}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the source file that defines `kernel` and of the shared device helpers."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_moe_dispatch_04_b200", "csrc")
    for name in (KERNEL_SOURCES[kernel], "common.cuh", "async.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current sources of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload, {}).get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# The CPU oracle as a timed baseline.

def oracle_chain_timed(inputs: dict, sample_tokens: int) -> tuple[float, int]:
    """Times the oracle's calls on the first `sample_tokens` tokens of the workload
    (expert stand-ins excluded). Returns (seconds, tokens)."""
    import oracle

    wl = inputs["workload"]
    n = min(sample_tokens, wl.bs)
    sub = wl.scaled(bs=n, a_capacity_override=0)
    inp = dict(inputs)
    inp["workload"] = sub
    for key in ("topk_idx", "topk_weights", "x", "mask", "shared", "grad_out"):
        if inp.get(key) is not None:
            inp[key] = np.ascontiguousarray(inp[key][:n])
    inp["ori_x"] = inp["x"] if inputs.get("ori_x") is not None else None
    if inp.get("expert_factor") is not None:
        inp["expert_factor"] = np.ascontiguousarray(inp["expert_factor"][:sub.a_capacity])
    secs = 0.0
    t = time.perf_counter()
    counts, send, assist, _ = oracle.dispatch_layout(inp["topk_idx"], sub.num_experts, sub.n_ids,
                                                     sub.a_capacity, inp["mask"])
    if sub.quant_mode == 2:
        if sub.smooth:
            q, sc = oracle.dispatch_permute_quant_smooth(inp["x"], inp["topk_idx"], inp["smooth"],
                                                         assist, sub.a_capacity, sub.dtype)
        else:
            q, sc = oracle.dispatch_permute_quant(inp["x"], assist, sub.k, sub.a_capacity,
                                                  sub.dtype)
        secs += time.perf_counter() - t
        y = workloads.expert_forward(inp, q, sc)
    else:
        ex = oracle.dispatch_permute(inp["x"], assist, sub.k, sub.a_capacity)
        secs += time.perf_counter() - t
        y = workloads.expert_forward(inp, ex)
    t = time.perf_counter()
    oracle.combine_fwd(y, inp["topk_idx"], inp["topk_weights"], assist,
                       num_experts=sub.num_experts, a_capacity=sub.a_capacity, dtype=sub.dtype,
                       zero_expert_num=sub.zero_expert_num, copy_expert_num=sub.copy_expert_num,
                       const_expert_num=sub.const_expert_num, mask=inp["mask"],
                       shared=inp["shared"], ori_x=inp["ori_x"], alpha1=inp["alpha1"],
                       alpha2=inp["alpha2"], const_v=inp["v"])
    if sub.backward:
        ge, _, _ = oracle.combine_bwd(inp["grad_out"], y, inp["topk_weights"], assist, k=sub.k,
                                      a_capacity=sub.a_capacity, dtype=sub.dtype, mask=inp["mask"])
        oracle.dispatch_bwd(ge, assist, bs=sub.bs, k=sub.k, a_capacity=sub.a_capacity,
                            dtype=sub.dtype, mask=inp["mask"])
    secs += time.perf_counter() - t
    return secs, n


def _oracle_leg(inputs: dict, sample: int, budget_s: float) -> tuple[float, int, float, int]:
    total_s, total_tok, passes = 0.0, 0, 0
    while total_s < budget_s and passes < 50:
        s, n = oracle_chain_timed(inputs, sample)
        total_s += s
        total_tok += n
        passes += 1
    return total_tok / total_s, passes, total_s, total_tok


def cpu_baseline(inputs: dict, budget_s: float = 10.0) -> dict:
    """The oracle timed on this host: single-threaded (the pinned build, the
    reported value) on a 2048-token sample, and its OpenMP build on all cores over
    the whole batch."""
    import oracle

    wl = inputs["workload"]
    sample = min(wl.bs, 2048)
    value, passes, secs, _ = _oracle_leg(inputs, sample, budget_s)
    steps_desc = (f"layout, permute, combine fwd"
                  f"{', combine bwd, dispatch bwd' if wl.backward else ''}")
    out = {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "sample": f"{passes} passes of the first {sample} tokens of {wl.name} through the "
                     f"single-threaded C++ oracle ({steps_desc}); {secs:.1f} s of CPU time"}
    nproc = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    with oracle.all_cores():
        threads = oracle.num_threads()
        v_all, p_all, s_all, _ = _oracle_leg(inputs, wl.bs, budget_s)
    out["all_cores"] = {"value": v_all, "unit": "tokens/s", "cores": threads, "nproc": nproc,
                        "kind": "oracle (OpenMP build, tokens split over threads)",
                        "sample": f"{p_all} passes of all {wl.bs} tokens of {wl.name} "
                                  f"({steps_desc}); {s_all:.1f} s wall"}
    return out


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inputs = workloads.generate(wl)
    # each step: a sample of tokens sized to about a quarter of a second of CPU work
    probe_s, probe_n = oracle_chain_timed(inputs, 64)
    sample = int(max(16, min(512, 0.25 / max(probe_s / probe_n, 1e-9))))
    for _ in range(args.warmup):
        oracle_chain_timed(inputs, sample)
    total_s, total_tok = 0.0, 0
    for _ in range(args.steps):
        s, n = oracle_chain_timed(inputs, sample)
        total_s += s
        total_tok += n
    value = total_tok / total_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "bs": wl.bs, "h": wl.h, "k": wl.k,
                       "num_experts": wl.num_experts, "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: the first {sample} tokens of {wl.name} "
                                       "through the single-threaded C++ oracle"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# One workload on the GPU: inputs resident in HBM, the path's calls, timing.

class Bench:
    """Builds one workload's resident inputs and the step's list of C-ABI calls."""

    def __init__(self, wl, args, dev, rank):
        import torch

        import combine_moe_dispatch_04_b200 as moe

        self.wl, self.args, self.dev = wl, args, dev
        self.torch, self.moe = torch, moe
        self.stream = torch.cuda.current_stream()
        self.inputs = inputs = workloads.generate(wl, seed=wl.seed + 1000 * rank)
        dt = wl.dtype
        tdt = torch.bfloat16 if dt == "bf16" else torch.float16

        def up(a):
            if a is None:
                return None
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).to(dev).view(tdt)
            return torch.from_numpy(a).to(dev)

        def down16(t):
            return t.cpu().view(torch.int16).numpy().view(np.uint16)

        sh = moe.Shape(bs=wl.bs, k=wl.k, h=wl.h, num_experts=wl.num_experts,
                       zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
                       const_expert_num=wl.const_expert_num, a_capacity=wl.a_capacity,
                       dtype=workloads.DTYPE_CODES[dt], mask_ndim=wl.mask_ndim)
        d = {k: up(inputs[k]) for k in ("topk_idx", "topk_weights", "x", "mask", "shared",
                                         "ori_x", "alpha1", "alpha2", "v", "grad_out",
                                         "smooth")}
        ws = moe.layout_workspace(sh, dev)
        lay = moe.dispatch_layout(sh, d["topk_idx"], d["mask"], workspace=ws)
        qm = wl.quant_mode
        if wl.smooth:
            expand, scales = moe.dispatch_permute_smooth(sh, d["x"], d["topk_idx"], lay,
                                                         d["smooth"])
        else:
            expand, scales = moe.dispatch_permute(sh, d["x"], lay, qm)
        torch.cuda.synchronize()
        r = int(lay.ep_send_counts[-1].item())
        # untimed expert stand-ins, computed once on the host from the GPU's dispatch output
        if qm == 2:
            y_host = workloads.expert_forward(inputs, expand.cpu().numpy(), scales.cpu().numpy())
        else:
            y_host = workloads.expert_forward(inputs, down16(expand))
        y = up(y_host)
        out = moe.combine_fwd(sh, y, d["topk_idx"], d["topk_weights"], lay,
                              x_active_mask=d["mask"], shared_expert_x=d["shared"],
                              ori_x=d["ori_x"], const_alpha_1=d["alpha1"],
                              const_alpha_2=d["alpha2"], const_v=d["v"])
        gexp = gw = gin = gx = None
        if wl.backward:
            gexp, gw = moe.combine_bwd(sh, d["grad_out"], y, d["topk_weights"], lay,
                                       x_active_mask=d["mask"])
            torch.cuda.synchronize()
            gin = up(workloads.expert_backward(inputs, down16(gexp)))
            gx = moe.dispatch_bwd(sh, gin, lay, x_active_mask=d["mask"])
        torch.cuda.synchronize()

        ori_tokens = 0
        if wl.copy_expert_num + wl.const_expert_num:
            ids = inputs["topk_idx"]
            lo = wl.num_experts + wl.zero_expert_num
            ori_tokens = int(np.any(ids >= lo, axis=1).sum())
        self.r = r
        bytes_per = byte_model(wl, r, ori_tokens)
        kernels = [k for k in KERNELS if k in bytes_per]
        sp_ws = sp_out = None
        if "combine_bwd_special" in bytes_per:
            n_ws = moe.moe_combine_bwd_special_workspace_bytes(ctypes.byref(sh.c()))
            sp_ws = torch.empty(max(n_ws, 16), dtype=torch.uint8, device=dev) if n_ws else None
            _, *sp_out = moe.combine_bwd_special(
                sh, d["grad_out"], d["topk_idx"], d["topk_weights"], d["ori_x"],
                x_active_mask=d["mask"], const_alpha_1=d["alpha1"], const_alpha_2=d["alpha2"],
                const_v=d["v"], grad_w=gw, workspace=sp_ws)
            torch.cuda.synchronize()

        # the step's results the caller reads back (swapped per slot by the e2e loop)
        o = {"out": out}
        if wl.backward:
            o.update(gw=gw, gx=gx)
        cq = args.combine_comm_quant
        q8_ws = None
        if cq == 2:  # the int8 combine's workspace, allocated once outside the timed steps
            nb = moe.moe_combine_fwd_comm_quant_workspace_bytes(ctypes.byref(sh.c()))
            q8_ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        special_ids = wl.zero_expert_num + wl.copy_expert_num + wl.const_expert_num
        self.q8_two_pass = (cq == 2 and special_ids == 0 and
                            wl.h // 8 >= 32 * (4 if wl.k <= 2 else 2 if wl.k <= 4 else 1))
        # the profiled kernel differs with the combine's quantisation mode
        self.traffic_key = wl.name + ("+comm_quant2" if cq == 2 else "")
        fused = args.fused_dispatch
        if fused:
            calls = [("dispatch", lambda st: moe.dispatch(
                sh, d["topk_idx"], d["x"], x_active_mask=d["mask"], comm_quant_mode=qm,
                workspace=ws, layout=lay, expand_x=expand, dynamic_scales=scales, stream=st))]
            bytes_per["dispatch"] = bytes_per.pop("layout") + bytes_per.pop("permute")
            kernels = ["dispatch"] + [k for k in kernels if k not in ("layout", "permute")]
        else:
            calls = [
                ("layout", lambda st: moe.dispatch_layout(sh, d["topk_idx"], d["mask"],
                                                       workspace=ws, out=lay, stream=st)),
                ("permute", lambda st: moe.dispatch_permute(sh, d["x"], lay, qm, expand_x=expand,
                                                         dynamic_scales=scales, stream=st)),
            ]
            if wl.smooth:
                calls[1] = ("permute", lambda st: moe.dispatch_permute_smooth(
                    sh, d["x"], d["topk_idx"], lay, d["smooth"], expand_x=expand,
                    dynamic_scales=scales, stream=st))
        calls += [
            ("combine_fwd", lambda st: moe.combine_fwd(
                sh, y, d["topk_idx"], d["topk_weights"], lay, x_active_mask=d["mask"],
                shared_expert_x=d["shared"], ori_x=d["ori_x"], const_alpha_1=d["alpha1"],
                const_alpha_2=d["alpha2"], const_v=d["v"], comm_quant_mode=cq, workspace=q8_ws,
                out=o["out"], stream=st)),
        ]
        if wl.backward:
            calls += [
                ("combine_bwd", lambda st: moe.combine_bwd(
                    sh, d["grad_out"], y, d["topk_weights"], lay, x_active_mask=d["mask"],
                    comm_quant_mode=cq, grad_expand=gexp, grad_w=o["gw"], stream=st)),
            ]
            if "combine_bwd_special" in bytes_per:
                calls += [("combine_bwd_special", lambda st: moe.combine_bwd_special(
                    sh, d["grad_out"], d["topk_idx"], d["topk_weights"], d["ori_x"],
                    x_active_mask=d["mask"], const_alpha_1=d["alpha1"],
                    const_alpha_2=d["alpha2"], const_v=d["v"], grad_w=o["gw"],
                    workspace=sp_ws, out=sp_out, stream=st))]
            calls += [
                ("dispatch_bwd", lambda st: moe.dispatch_bwd(sh, gin, lay,
                                                          x_active_mask=d["mask"],
                                                          grad_x=o["gx"], stream=st)),
            ]
        self.d, self.o, self.calls = d, o, calls
        self.bytes_per, self.kernels = bytes_per, kernels
        # the kernel that moves the most bytes; the timed steps bracket it with events
        self.dominant = max((k for k in kernels if k not in ("layout", "dispatch")),
                            key=lambda k: bytes_per[k])
        if fused and wl.bs <= 1024 and qm == 0:
            dispatch_launches = 1
        else:
            dispatch_launches = layout_launches(wl.bs, wl.num_experts, wl.k) + 1
        special_bwd_launches = 0
        if "combine_bwd_special" in bytes_per:
            special_bwd_launches = 1 + (2 if wl.const_expert_num else 0)
        self.launches_per_step = (dispatch_launches + (2 if self.q8_two_pass else 1)
                                  + (2 if wl.backward else 0) + special_bwd_launches)
        self.use_graph = not args.no_graph
        self.plain_graph = self.capture() if self.use_graph else None

    # ---- launching

    def run_calls(self, st, marks=None):
        for name, fn in self.calls:
            if marks is not None and name in marks:
                marks[name][0].record(st)
            fn(st)
            if marks is not None and name in marks:
                marks[name][1].record(st)

    def new_marks(self, names, external=False):
        torch = self.torch
        ev = lambda: torch.cuda.Event(enable_timing=True, external=external)  # noqa: E731
        m = {"start": ev(), "end": ev()}
        for n_ in names:
            m[n_] = (ev(), ev())
        return m

    def capture(self, marks=None):
        """A CUDA graph of the step's launches (programmatic-launch edges kept), with
        event-record nodes around the kernels named in `marks`."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run_calls(torch.cuda.current_stream(), marks)
        return g

    def step(self, marks=None, graph=None):
        """One pass of the path. `marks` maps "start"/"end" to an event and kernel
        names to (before, after) event pairs; kernels without events keep their
        programmatic-launch overlap with their neighbours. With `graph`, the pass
        is that captured graph (whose own events are already inside)."""
        if marks is not None:
            marks["start"].record(self.stream)
        if graph is not None:
            graph.replay()
        else:
            self.run_calls(self.stream, marks)
        if marks is not None:
            marks["end"].record(self.stream)

    # ---- timing

    def timed_run(self, steps, warmup, flush_l2, world, sampler=None):
        """W warm-up steps, then `steps` timed steps (an L2 flush before each, outside
        the step's events), each carrying only its own start/end events; then, in the
        same bracketed window, ceil(steps / DOM_EVERY) more steps with events around
        the dominant kernel as well (an event between two kernels costs both their
        launch overlap, so those steps are kept out of the step statistics)."""
        import torch.distributed as dist
        torch = self.torch
        dom = self.dominant
        for _ in range(warmup):
            flush_l2()
            self.step(graph=self.plain_graph)
        torch.cuda.synchronize()
        n_dom = max(1, -(-steps // DOM_EVERY))
        marks = [self.new_marks([]) for _ in range(steps)]
        dmarks = [self.new_marks([dom], external=self.use_graph) for _ in range(n_dom)]
        dgraphs = [self.capture({dom: m[dom]}) if self.use_graph else None for m in dmarks]
        if self.use_graph:
            for g in dgraphs:  # warm every graph once
                flush_l2()
                self.step(graph=g)
            torch.cuda.synchronize()
        if sampler is not None:
            sampler.start()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        for i in range(steps):
            flush_l2()
            self.step({"start": marks[i]["start"], "end": marks[i]["end"]},
                      graph=self.plain_graph)
        for i in range(n_dom):
            flush_l2()
            if self.use_graph:
                self.step({"start": dmarks[i]["start"], "end": dmarks[i]["end"]},
                          graph=dgraphs[i])
            else:
                self.step(dmarks[i])
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t1 = time.time()
        clocks = sampler.stop(t0, t1) if sampler is not None else None
        step_ms = [m["start"].elapsed_time(m["end"]) for m in marks]
        dom_ms = [m[dom][0].elapsed_time(m[dom][1]) for m in dmarks]
        del dgraphs
        return step_ms, dom_ms, clocks

    def accepted_run(self, steps, warmup, flush_l2, world, rank, uuid):
        """Runs until std/mean of the kept steps is at most ACCEPT_CV (max over ranks),
        at most MAX_RUNS times; returns the run with the smallest std/mean."""
        best = None
        runs = 0
        for _ in range(MAX_RUNS):
            sampler = ClockSampler(uuid) if rank == 0 else None
            step_ms, dom_ms, clocks = self.timed_run(steps, warmup, flush_l2, world, sampler)
            runs += 1
            st = trimmed_stats(step_ms)
            cv = reduce_max(st["cv"])
            mean = reduce_max(st["mean"])
            if best is None or cv < best["cv"]:
                best = {"cv": cv, "mean_ms": mean, "stats": st, "step_ms": step_ms,
                        "dom_ms": dom_ms, "clocks": clocks}
            if cv <= ACCEPT_CV:
                break
        best["runs"] = runs
        best["accepted"] = best["cv"] <= ACCEPT_CV
        return best

    def kernel_diagnostic(self, flush_l2, n):
        """Separate untimed steps with events around every kernel (each loses its
        launch overlap): per-kernel means in microseconds."""
        torch = self.torch
        diag = [self.new_marks(self.kernels) for _ in range(n)]
        for m in diag:
            flush_l2()
            self.step(m)
        torch.cuda.synchronize()
        return {k: 1e3 * statistics.fmean(m[k][0].elapsed_time(m[k][1]) for m in diag)
                for k in self.kernels}

    def summary(self, run, peak):
        """Throughput and roofline figures of one accepted run."""
        wl = self.wl
        ms = run["mean_ms"]
        bytes_step = sum(self.bytes_per.values())
        gbs = bytes_step / (ms * 1e-3) / 1e9
        dom = self.dominant
        dom_us = 1e3 * statistics.fmean(run["dom_ms"]) if run["dom_ms"] else float("nan")
        ach = self.bytes_per[dom] / (dom_us * 1e-6) / 1e9
        return {
            "ms_per_step": ms, "tokens_per_s": wl.bs / (ms * 1e-3),
            "hbm_gbs": round(gbs, 1), "hbm_frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
            "hbm_frac_of_measured": round(gbs / peak, 4),
            "algorithmic_bytes_per_step": bytes_step,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(ach / peak, 4),
                         "algorithmic_bytes": self.bytes_per[dom],
                         "us_per_launch": round(dom_us, 3)},
            "std_over_mean": round(run["cv"], 5), "accepted": run["accepted"],
            "runs": run["runs"], "clocks": run["clocks"],
        }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="moe", choices=["moe", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--fused-dispatch", action="store_true",
                    help="layout + permute through the single moe_dispatch call")
    ap.add_argument("--combine-comm-quant", type=int, default=0, choices=[0, 2],
                    help="combine forward with comm_quant_mode 2 (int8 round trip)")
    ap.add_argument("--with-backward", action="store_true",
                    help="add the backward steps to a forward-only workload")
    ap.add_argument("--smooth-quant", action="store_true",
                    help="int8 dispatch of x * smooth_scales[e] (int8 workloads only)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step eagerly instead of replaying a CUDA graph of it")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--per-config-steps", type=int, default=100)
    args = ap.parse_args()
    wl = workloads.BY_NAME[args.workload]
    if args.with_backward and not wl.backward:
        wl = wl.scaled(backward=True, name=wl.name + "+backward")
    if args.smooth_quant:
        if wl.quant_mode != 2 or args.fused_dispatch:
            ap.error("--smooth-quant needs an int8 workload and the separate permute call")
        wl = wl.scaled(smooth=True, name=wl.name + "+smooth")
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        # replicas: a host-side group for the barrier and the timing max only
        dist.init_process_group("gloo", timeout=_dt.timedelta(seconds=120))
    dev = torch.device("cuda", local)

    # L2 flush between steps: write a buffer twice the size of L2, then read another
    # one as large, so the step starts with none of its data in L2 and without the
    # flush's dirty lines, whose write-back would otherwise be billed to the step.
    # Both run before the step's start event.
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20)
    flush = torch.empty(2 * l2 // 4, dtype=torch.int32, device=dev)
    sweep = torch.zeros(2 * l2 // 4, dtype=torch.float32, device=dev)
    sweep_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        torch.sum(sweep, dim=0, out=sweep_out)  # one reduction kernel

    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    peak, peak_kind = measured_hbm_peak()

    b = Bench(wl, args, dev, rank)
    run = b.accepted_run(args.steps, args.warmup, flush_l2, world, rank, uuid)
    ms_per_step = run["mean_ms"]
    value = whole_job_throughput(wl.bs, 1, world, ms_per_step)
    per_kernel_us = b.kernel_diagnostic(flush_l2, min(args.steps, 20))

    # e2e: pinned host inputs -> H2D -> the path through the C ABI -> D2H of the results,
    # every step. Inputs and results are double-buffered on the device: step i's
    # uploads (a copy stream) and step i-1's read-back (another) overlap step i-1's
    # and step i's kernels, as a serving loop would run them.
    e2e = None
    if not args.no_e2e:
        d, o, stream = b.d, b.o, b.stream
        in_keys = [k for k in ("topk_idx", "topk_weights", "x", "mask", "shared", "grad_out")
                   if d[k] is not None]
        h_in = {k: d[k].cpu().pin_memory() for k in in_keys}
        out_keys = list(o)
        h_out = {k: o[k].cpu().pin_memory() for k in out_keys}
        bi = sum(t.numel() * t.element_size() for t in h_in.values())
        bo = sum(t.numel() * t.element_size() for t in h_out.values())
        e2e_steps = max(3, args.steps // 4)
        slots = [({k: d[k] for k in in_keys}, dict(o)),
                 ({k: torch.empty_like(d[k]) for k in in_keys},
                  {k: torch.empty_like(o[k]) for k in out_keys})]
        up_s, down_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev = [{n: torch.cuda.Event() for n in ("in", "done", "read")} for _ in slots]
        uses_ori = d["ori_x"] is not None

        def e2e_step(i):
            din, dout = slots[i % 2]
            e = ev[i % 2]
            with torch.cuda.stream(up_s):
                if i >= 2:
                    up_s.wait_event(e["done"])  # step i-2 no longer reads these inputs
                for k in in_keys:
                    din[k].copy_(h_in[k], non_blocking=True)
                e["in"].record(up_s)
            stream.wait_event(e["in"])
            if i >= 2:
                stream.wait_event(e["read"])  # step i-2's results have been read back
            d.update(din)
            if uses_ori:
                d["ori_x"] = din["x"]  # the token rows the copy/const experts return
            o.update(dout)
            b.step()
            e["done"].record(stream)
            with torch.cuda.stream(down_s):
                down_s.wait_event(e["done"])
                for k in out_keys:
                    h_out[k].copy_(dout[k], non_blocking=True)
                e["read"].record(down_s)

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        ea = torch.cuda.Event(enable_timing=True)
        eb = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        ea.record(stream)
        up_s.wait_stream(stream)
        down_s.wait_stream(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        stream.wait_stream(down_s)
        eb.record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max(ea.elapsed_time(eb))
        e2e = {"value": whole_job_throughput(wl.bs, e2e_steps, world, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": e2e_steps,
               "note": "double-buffered: each step's uploads and read-back overlap the "
                       "neighbouring steps' kernels on two copy streams; eager launches "
                       "through the binding"}
        # the timed graphs captured the original buffers: restore them
        d.update(slots[0][0])
        if uses_ori:
            d["ori_x"] = slots[0][0]["x"]
        o.update(slots[0][1])

    head = b.summary(run, peak)
    launches = b.launches_per_step
    line_extra = {"dominant": b.dominant, "traffic_key": b.traffic_key, "r": b.r,
                  "q8_two_pass": b.q8_two_pass, "kernels": b.kernels,
                  "bytes_per": b.bytes_per, "use_graph": b.use_graph}
    inputs_head = b.inputs
    del b
    torch.cuda.empty_cache()

    # Every workload, same process and method (fewer steps), for the per-config block.
    per_config = {}
    if not args.no_per_config:
        for w in workloads.WORKLOADS:
            if w.name == wl.name and not (args.fused_dispatch or args.combine_comm_quant):
                per_config[w.name] = {k: head[k] for k in (
                    "ms_per_step", "tokens_per_s", "hbm_gbs", "hbm_frac_of_8tbs",
                    "hbm_frac_of_measured", "roofline", "std_over_mean", "accepted", "runs",
                    "clocks")}
            else:
                pc_args = argparse.Namespace(**vars(args))
                # small batches take the one-launch dispatch (layout + permute), the
                # library's call for them; the others the two calls
                pc_args.fused_dispatch = w.bs <= FUSED_DISPATCH_MAX_TOKENS
                pc_args.combine_comm_quant = 0
                bw = Bench(w, pc_args, dev, rank)
                rw = bw.accepted_run(args.per_config_steps, args.warmup, flush_l2, world, rank,
                                     uuid)
                per_config[w.name] = bw.summary(rw, peak)
                per_config[w.name]["fused_dispatch"] = pc_args.fused_dispatch
                del bw
                torch.cuda.empty_cache()
            pc = per_config[w.name]
            pc["meets_70pct_of_8tbs"] = (None if w.name.startswith("tiny")
                                         else pc["hbm_frac_of_8tbs"] >= TARGET_FRAC_OF_8TBS)

    if rank == 0:
        kstats = {}
        for k in line_extra["kernels"]:
            us = per_kernel_us[k]
            kstats[k] = {"us": round(us, 3), "bytes": line_extra["bytes_per"][k],
                         "gbs": round(line_extra["bytes_per"][k] / (us * 1e-6) / 1e9, 1)}
        roof = dict(head["roofline"])
        roof.update(peak_kind=peak_kind,
                    traffic=profiled_traffic(line_extra["dominant"], line_extra["traffic_key"]),
                    timed=f"CUDA events around this kernel in ceil(steps / {DOM_EVERY}) more steps "
                          f"({len(run['dom_ms'])} launches)")
        st = run["stats"]
        cq = args.combine_comm_quant
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": "synthetic",
            "config": {"workload": wl.name, "bs": wl.bs, "h": wl.h, "k": wl.k,
                       "num_experts": wl.num_experts, "routed_pairs": line_extra["r"],
                       "a_capacity": wl.a_capacity, "parallelism": "replicas",
                       "fused_dispatch": bool(args.fused_dispatch),
                       "smooth_quant": bool(wl.smooth),
                       "combine_comm_quant_mode": cq,
                       "combine_int8_kernels": ("two-pass" if line_extra["q8_two_pass"]
                                                else "single-pass") if cq == 2 else None,
                       "launch": ("CUDA graph of the step" if line_extra["use_graph"]
                                  else "eager launches"),
                       "l2": "flushed before every step (write of 2x L2, then a read of another "
                             "2x L2 so no dirty flush lines are written back inside the step), "
                             "outside the step events",
                       "statistics": f"value and ms_per_step: mean of the K timed steps (each "
                                     f"with only its start/end events) without the {DROP_TOP} "
                                     f"slowest, max over ranks; accepted when "
                                     f"std/mean <= {ACCEPT_CV:.0%}, else rerun (at most "
                                     f"{MAX_RUNS} runs, the steadiest kept)"},
            "hbm_gbs": head["hbm_gbs"], "hbm_frac_of_8tbs": head["hbm_frac_of_8tbs"],
            "hbm_frac_of_measured": head["hbm_frac_of_measured"],
            "algorithmic_bytes_per_step": head["algorithmic_bytes_per_step"],
            "roofline": roof,
            "kernels_diagnostic": {"note": "separate untimed steps with events around every "
                                           "kernel (no launch overlap)", **kstats},
            "gpu_launches": launches * (args.steps + len(run["dom_ms"])),
            "e2e": e2e,
            "clocks": run["clocks"],
            "step_ms_stats": {"trimmed_mean_drop_top3": st["mean"], "std": st["std"],
                              "std_over_mean": st["cv"], "plain_mean": st["plain_mean"],
                              "median": st["median"], "min": st["min"], "max": st["max"],
                              "runs": run["runs"], "accepted": run["accepted"]},
            "per_config": per_config or None,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(inputs_head)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
