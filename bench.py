"""Benchmark of the MoE dispatch + combine forward + backward path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  moe_dispatch_layout -> moe_dispatch_permute -> moe_combine_fwd -> moe_combine_bwd
  -> moe_dispatch_bwd
(forward-only workloads stop after moe_combine_fwd). The experts between dispatch and
combine are outside the path: their outputs (and input gradients) are computed once,
untimed, and stay resident in HBM like every other input.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on the host cores

Prints one JSON line (rank 0). Multi-GPU runs are independent replicas (one process
per GPU, launched with torch.distributed.run); only the barrier and the max-over-ranks
timing use the process group.
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
DEFAULT_WORKLOAD = "uniform_bs8192_h1536_k8_e64"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
KERNELS = ("layout", "permute", "combine_fwd", "combine_bwd", "combine_bwd_special",
           "dispatch_bwd")
DOM_EVERY = 4


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
# Replicas: only the timing is reduced across ranks (max), never data.

def reduce_max(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(tokens_per_rank_step: int, steps: int, world: int,
                         max_total_ms: float) -> float:
    """Tokens of all replicas divided by the slowest replica's time."""
    return tokens_per_rank_step * steps * world / (max_total_ms * 1e-3)


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

def moe_layout_small_max_tokens() -> int:
    """Largest BS the layout handles in one launch (one CTA); above it, two launches."""
    return 1024


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


def oracle_chain_timed(inputs: dict, sample_tokens: int) -> tuple[float, int]:
    """Times the oracle's five calls on the first `sample_tokens` tokens of the
    workload (expert stand-ins excluded). Returns (seconds, tokens)."""
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


def cpu_baseline(inputs: dict, budget_s: float = 10.0) -> dict:
    wl = inputs["workload"]
    sample = min(wl.bs, 2048)
    total_s, total_tok, passes = 0.0, 0, 0
    while total_s < budget_s and passes < 50:
        s, n = oracle_chain_timed(inputs, sample)
        total_s += s
        total_tok += n
        passes += 1
    return {"value": total_tok / total_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{passes} passes of the first {sample} tokens of {wl.name} through the "
                      f"single-threaded C++ oracle (layout, permute, combine fwd"
                      f"{', combine bwd, dispatch bwd' if wl.backward else ''}); "
                      f"{total_s:.1f} s of CPU time"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inputs = workloads.generate(wl)
    sample = min(wl.bs, 512)
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
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
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

    import combine_moe_dispatch_04_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    inputs = workloads.generate(wl, seed=wl.seed + 1000 * rank)
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
    d = {k: up(inputs[k]) for k in ("topk_idx", "topk_weights", "x", "mask", "shared", "ori_x",
                                     "alpha1", "alpha2", "v", "grad_out", "smooth")}
    ws = moe.layout_workspace(sh, dev)
    lay = moe.dispatch_layout(sh, d["topk_idx"], d["mask"], workspace=ws)
    qm = wl.quant_mode
    if wl.smooth:
        expand, scales = moe.dispatch_permute_smooth(sh, d["x"], d["topk_idx"], lay, d["smooth"])
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
    out = moe.combine_fwd(sh, y, d["topk_idx"], d["topk_weights"], lay, x_active_mask=d["mask"],
                          shared_expert_x=d["shared"], ori_x=d["ori_x"],
                          const_alpha_1=d["alpha1"], const_alpha_2=d["alpha2"],
                          const_v=d["v"])
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
    q8_two_pass = (cq == 2 and special_ids == 0 and
                   wl.h // 8 >= 32 * (4 if wl.k <= 2 else 2 if wl.k <= 4 else 1))
    # the profiled kernel differs with the combine's quantisation mode
    traffic_key = wl.name + ("+comm_quant2" if cq == 2 else "")
    if args.fused_dispatch:
        calls = [("dispatch", lambda st: moe.dispatch(
            sh, d["topk_idx"], d["x"], x_active_mask=d["mask"], comm_quant_mode=qm,
            workspace=ws, layout=lay, expand_x=expand, dynamic_scales=scales, stream=st))]
        bytes_per["dispatch"] = bytes_per.pop("layout") + bytes_per.pop("permute")
        kernels = ["dispatch"] + [k for k in kernels if k not in ("layout", "permute")]
    else:
        calls = [
            ("layout", lambda st: moe.dispatch_layout(sh, d["topk_idx"], d["mask"], workspace=ws,
                                                   out=lay, stream=st)),
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
                grad_expand=gexp, grad_w=o["gw"], stream=st)),
        ]
        if "combine_bwd_special" in bytes_per:
            calls += [("combine_bwd_special", lambda st: moe.combine_bwd_special(
                sh, d["grad_out"], d["topk_idx"], d["topk_weights"], d["ori_x"],
                x_active_mask=d["mask"], const_alpha_1=d["alpha1"], const_alpha_2=d["alpha2"],
                const_v=d["v"], grad_w=o["gw"], workspace=sp_ws, out=sp_out, stream=st))]
        calls += [
            ("dispatch_bwd", lambda st: moe.dispatch_bwd(sh, gin, lay, x_active_mask=d["mask"],
                                                      grad_x=o["gx"], stream=st)),
        ]
    # the kernel that moves the most bytes; the timed steps bracket it with events
    dominant = max((k for k in kernels if k not in ("layout", "dispatch")),
                   key=lambda k: bytes_per[k])

    def run_calls(st, marks=None):
        for name, fn in calls:
            if marks is not None and name in marks:
                marks[name][0].record(st)
            fn(st)
            if marks is not None and name in marks:
                marks[name][1].record(st)

    def new_marks(names, external=False):
        ev = lambda: torch.cuda.Event(enable_timing=True, external=external)  # noqa: E731
        m = {"start": ev(), "end": ev()}
        for n_ in names:
            m[n_] = (ev(), ev())
        return m

    # CUDA graphs of the step: one plain, and one per sampled step with timing
    # events (graph event-record nodes) around the dominant kernel.
    graphs = {}

    def capture(marks=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run_calls(torch.cuda.current_stream(), marks)
        return g

    def step(marks=None, graph=None):
        """One pass of the path. `marks` maps "start"/"end" to an event and kernel
        names to (before, after) event pairs; kernels without events keep their
        programmatic-launch overlap with their neighbours. With `graph`, the
        pass is that captured graph (whose own events are already inside)."""
        if marks is not None:
            marks["start"].record(stream)
        if graph is not None:
            graph.replay()
        else:
            run_calls(stream, marks)
        if marks is not None:
            marks["end"].record(stream)

    tiled = wl.bs > moe_layout_small_max_tokens()
    if args.fused_dispatch and not tiled and qm == 0:
        dispatch_launches = 1
    else:
        dispatch_launches = (2 if tiled else 1) + 1
    special_bwd_launches = 0
    if "combine_bwd_special" in bytes_per:
        special_bwd_launches = 1 + (2 if wl.const_expert_num else 0)
    launches_per_step = (dispatch_launches + (2 if q8_two_pass else 1) + (2 if wl.backward else 0)
                         + special_bwd_launches)

    # L2 flush between steps: write a buffer twice the size of L2, then read
    # another one as large, so the step starts with none of its data in L2 and
    # without the flush's dirty lines, whose write-back would otherwise be
    # billed to the step. Both run before the step's start event.
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20)
    flush = torch.empty(2 * l2 // 4, dtype=torch.int32, device=dev)
    sweep = torch.zeros(2 * l2 // 4, dtype=torch.float32, device=dev)
    sweep_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        torch.sum(sweep, dim=0, out=sweep_out)  # one reduction kernel

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()

    # Every DOM_EVERY-th timed step also brackets the dominant kernel with events
    # (an event between two kernels costs both their launch overlap, so the
    # other steps carry only the step's own start/end events).
    sampled = [i % DOM_EVERY == DOM_EVERY - 1 for i in range(args.steps)]
    use_graph = not args.no_graph
    marks, step_graphs = [], []
    if use_graph:
        plain = capture()
        for i in range(args.steps):
            m = new_marks([])
            if sampled[i]:
                inner = new_marks([dominant], external=True)
                m[dominant] = inner[dominant]
                step_graphs.append(capture({dominant: inner[dominant]}))
            else:
                step_graphs.append(plain)
            marks.append(m)
        for _ in range(2):  # warm the graphs
            flush_l2()
            step(graph=plain)
        torch.cuda.synchronize()
    else:
        marks = [new_marks([dominant] if sampled[i] else []) for i in range(args.steps)]
        step_graphs = [None] * args.steps
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid if rank == 0 else None)
    if rank == 0:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(args.steps):
        flush_l2()
        if step_graphs[i] is not None:
            step({"start": marks[i]["start"], "end": marks[i]["end"]}, graph=step_graphs[i])
        else:
            step(marks[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t1 = time.time()
    clocks = sampler.stop(t0, t1) if rank == 0 else None

    step_ms = [m["start"].elapsed_time(m["end"]) for m in marks]
    dom_ms = [m[dominant][0].elapsed_time(m[dominant][1]) for m in marks if dominant in m]
    total_ms = reduce_max(float(sum(step_ms)), dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_throughput(wl.bs, args.steps, world, total_ms)
    bytes_step = sum(bytes_per.values())

    # Per-kernel breakdown from separate diagnostic steps (not the timed ones):
    # events around every kernel, which costs each kernel its launch overlap.
    diag = [new_marks(kernels) for _ in range(min(args.steps, 20))]
    for m in diag:
        flush_l2()
        step(m)
    torch.cuda.synchronize()
    per_kernel_ms = {k: [m[k][0].elapsed_time(m[k][1]) for m in diag] for k in kernels}

    # e2e: pinned host inputs -> H2D -> the path through the C ABI -> D2H of the results,
    # every step. Inputs and results are double-buffered on the device: step i's
    # uploads (a copy stream) and step i-1's read-back (another) overlap step i-1's
    # and step i's kernels, as a serving loop would run them.
    e2e = None
    if not args.no_e2e:
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
            step()
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
        e_ms = reduce_max(ea.elapsed_time(eb), dev)
        e2e = {"value": whole_job_throughput(wl.bs, e2e_steps, world, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": e2e_steps,
               "note": "double-buffered: each step's uploads and read-back overlap the "
                       "neighbouring steps' kernels on two copy streams"}

    if rank == 0:
        peak, peak_kind = measured_hbm_peak()
        kstats = {}
        for k in kernels:
            us = 1e3 * statistics.fmean(per_kernel_ms[k])
            kstats[k] = {"us": round(us, 3), "bytes": bytes_per[k],
                         "gbs": round(bytes_per[k] / (us * 1e-6) / 1e9, 1)}
        dom = dominant
        dom_us = 1e3 * statistics.fmean(dom_ms)
        ach = round(bytes_per[dom] / (dom_us * 1e-6) / 1e9, 1)
        gbs = bytes_step / (ms_per_step * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dt,
            "data": "synthetic",
            "config": {"workload": wl.name, "bs": wl.bs, "h": wl.h, "k": wl.k,
                       "num_experts": wl.num_experts, "routed_pairs": r,
                       "a_capacity": wl.a_capacity, "parallelism": "replicas",
                       "fused_dispatch": bool(args.fused_dispatch),
                       "smooth_quant": bool(wl.smooth),
                       "combine_comm_quant_mode": cq,
                       "combine_int8_kernels": ("two-pass" if q8_two_pass else "single-pass")
                                               if cq == 2 else None,
                       "launch": "CUDA graph of the step" if use_graph else "eager launches",
                       "l2": "flushed before every step (write of 2x L2, then a read of another 2x L2 so "
                             "no dirty flush lines are written back inside the step), outside "
                             "the step events"},
            "hbm_gbs": round(gbs, 1), "hbm_frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
            "hbm_frac_of_measured": round(gbs / peak, 4),
            "algorithmic_bytes_per_step": bytes_step,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(ach / peak, 4),
                         "traffic": profiled_traffic(dom, traffic_key),
                         "algorithmic_bytes": bytes_per[dom], "us_per_launch": round(dom_us, 3),
                         "timed": f"CUDA events around this kernel in every {DOM_EVERY}th timed "
                                  f"step ({len(dom_ms)} launches)"},
            "kernels_diagnostic": {"note": "separate untimed steps with events around every "
                                           "kernel (no launch overlap)", **kstats},
            "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e,
            "clocks": clocks,
            "step_ms_stats": {"mean": statistics.fmean(step_ms),
                              "median": statistics.median(step_ms),
                              "trimmed_mean_drop_top3": statistics.fmean(
                                  sorted(step_ms)[:-3] if len(step_ms) > 6 else step_ms),
                              "std": statistics.pstdev(step_ms)},
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(inputs)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
