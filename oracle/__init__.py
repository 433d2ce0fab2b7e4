"""ctypes wrapper of the CPU oracle (``oracle/oracle.cpp``).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this module. The CUDA product path never does.

All 16-bit tensors are numpy ``uint16`` bit patterns (bf16 or fp16, per ``dtype``).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
LIB_PATH = os.path.join(_HERE, "liboracle.so")
# The same source built with -fopenmp: the per-token loops run on all host cores
# (results unchanged). Only the benchmark's all-cores CPU timing uses it; every
# test of the oracle runs the plain single-threaded build above.
LIB_OMP_PATH = os.path.join(_HERE, "liboracle_omp.so")
DTYPE_CODES = {"bf16": 0, "fp16": 1}


def build(force: bool = False, parallel: bool = False) -> str:
    """Compile the oracle with g++ (no FMA contraction, no fast-math); with
    parallel, the OpenMP build."""
    path = LIB_OMP_PATH if parallel else LIB_PATH
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", *(["-fopenmp"] if parallel else []), _SRC,
               "-o", path + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(path + ".tmp", path)
    return path


_libs: dict = {}
_parallel = False


@contextlib.contextmanager
def all_cores():
    """Within this block every oracle call runs the OpenMP build."""
    global _parallel
    prev, _parallel = _parallel, True
    try:
        yield
    finally:
        _parallel = prev


def num_threads() -> int:
    """Threads the active build runs its per-token loops on."""
    return int(lib().oracle_num_threads())


def lib():
    key = "omp" if _parallel else "plain"
    if key not in _libs:
        # ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        path = (build(parallel=True) if _parallel
                else os.environ.get("ORACLE_LIB") or build())
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = i
        L.oracle_decode16.argtypes = [ctypes.c_uint16, i]
        L.oracle_decode16.restype = ctypes.c_float
        L.oracle_encode16.argtypes = [ctypes.c_float, i]
        L.oracle_encode16.restype = ctypes.c_uint16
        L.oracle_decode16_array.argtypes = [P, P, ctypes.c_long, i]
        L.oracle_decode16_array.restype = None
        L.oracle_encode16_array.argtypes = [P, P, ctypes.c_long, i]
        L.oracle_encode16_array.restype = None
        L.oracle_dispatch_layout.argtypes = [i, i, i, i, i, P, P, i, P, P, P]
        L.oracle_dispatch_layout.restype = i
        L.oracle_dispatch_permute.argtypes = [i, i, i, i, P, P, P]
        L.oracle_dispatch_permute.restype = None
        L.oracle_dispatch_permute_quant.argtypes = [i, i, i, i, i, P, P, P, P]
        L.oracle_dispatch_permute_quant.restype = None
        L.oracle_dispatch_permute_quant_smooth.argtypes = [i, i, i, i, i, P, P, P, P, P, P]
        L.oracle_dispatch_permute_quant_smooth.restype = None
        L.oracle_combine_fwd.argtypes = [i, i, i, i, i, i, i, i, i, P, P, P, P, P, i,
                                         P, P, P, P, P, i, P]
        L.oracle_combine_fwd.restype = None
        L.oracle_combine_bwd.argtypes = [i, i, i, i, i, P, P, P, P, P, i, P, P, P]
        L.oracle_combine_bwd.restype = None
        L.oracle_combine_bwd_comm_quant.argtypes = [i, i, i, i, i, P, P, P, P, P, i, P, P, P]
        L.oracle_combine_bwd_comm_quant.restype = None
        L.oracle_combine_bwd_special.argtypes = [i, i, i, i, i, i, i, i, P, P, P, P, i, P, P, P,
                                                 P, P, P, P, P, P, P, P, P, P]
        L.oracle_combine_bwd_special.restype = None
        L.oracle_dispatch_bwd.argtypes = [i, i, i, i, i, P, P, P, i, P]
        L.oracle_dispatch_bwd.restype = None
        _libs[key] = L
    return _libs[key]


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dt):
    return None if a is None else np.ascontiguousarray(a, dtype=dt)


def decode16(bits: int, dtype: str) -> float:
    return lib().oracle_decode16(int(bits), DTYPE_CODES[dtype])


def encode16(f: float, dtype: str) -> int:
    return int(lib().oracle_encode16(float(f), DTYPE_CODES[dtype]))


def decode16_array(bits, dtype: str) -> np.ndarray:
    b = _c(bits, np.uint16)
    f = np.empty(b.shape, np.float32)
    lib().oracle_decode16_array(_p(b), _p(f), b.size, DTYPE_CODES[dtype])
    return f


def encode16_array(f, dtype: str) -> np.ndarray:
    a = _c(f, np.float32)
    b = np.empty(a.shape, np.uint16)
    lib().oracle_encode16_array(_p(a), _p(b), a.size, DTYPE_CODES[dtype])
    return b


def assist_elems(bs: int, k: int, a_capacity: int) -> int:
    return a_capacity + bs * k


def dispatch_layout(topk_idx, num_experts, n_ids, a_capacity, mask=None):
    """Returns (expert_token_nums (E,), ep_send_counts (E+1,), assist_info, status)."""
    idx = _c(topk_idx, np.int32)
    bs, k = idx.shape
    m = _c(mask, np.uint8)
    mask_ndim = 0 if m is None else m.ndim
    counts = np.zeros(num_experts, np.int32)
    send = np.zeros(num_experts + 1, np.int32)
    assist = np.zeros(assist_elems(bs, k, a_capacity), np.int32)
    st = lib().oracle_dispatch_layout(bs, k, num_experts, n_ids, a_capacity, _p(idx), _p(m),
                                      mask_ndim, _p(counts), _p(send), _p(assist))
    return counts, send, assist, int(st)


def dispatch_permute(x, assist_info, k, a_capacity):
    x = _c(x, np.uint16)
    bs, h = x.shape
    out = np.zeros((a_capacity, h), np.uint16)
    lib().oracle_dispatch_permute(bs, k, h, a_capacity, _p(x), _p(_c(assist_info, np.int32)),
                                  _p(out))
    return out


def dispatch_permute_quant(x, assist_info, k, a_capacity, dtype):
    x = _c(x, np.uint16)
    bs, h = x.shape
    q = np.zeros((a_capacity, h), np.int8)
    sc = np.zeros(a_capacity, np.float32)
    lib().oracle_dispatch_permute_quant(bs, k, h, a_capacity, DTYPE_CODES[dtype], _p(x),
                                        _p(_c(assist_info, np.int32)), _p(q), _p(sc))
    return q, sc


def dispatch_permute_quant_smooth(x, topk_idx, smooth_scales, assist_info, a_capacity, dtype):
    """int8 permute of x[t] * smooth_scales[e] per routed pair: (codes (A, H), scales (A,))."""
    x = _c(x, np.uint16)
    bs, h = x.shape
    idx = _c(topk_idx, np.int32)
    q = np.zeros((a_capacity, h), np.int8)
    sc = np.zeros(a_capacity, np.float32)
    lib().oracle_dispatch_permute_quant_smooth(
        bs, idx.shape[1], h, a_capacity, DTYPE_CODES[dtype], _p(x), _p(idx),
        _p(_c(smooth_scales, np.float32)), _p(_c(assist_info, np.int32)), _p(q), _p(sc))
    return q, sc


def combine_fwd(expand_x, topk_idx, topk_weights, assist_info, *, num_experts, a_capacity,
                dtype, zero_expert_num=0, copy_expert_num=0, const_expert_num=0,
                mask=None, shared=None, ori_x=None, alpha1=None, alpha2=None, const_v=None,
                comm_quant_mode=0):
    idx = _c(topk_idx, np.int32)
    bs, k = idx.shape
    ex = _c(expand_x, np.uint16)
    h = ex.shape[1]
    m = _c(mask, np.uint8)
    out = np.zeros((bs, h), np.uint16)
    args = [_c(shared, np.uint16), _c(ori_x, np.uint16), _c(alpha1, np.uint16),
            _c(alpha2, np.uint16), _c(const_v, np.uint16)]
    lib().oracle_combine_fwd(bs, k, h, num_experts, zero_expert_num, copy_expert_num,
                             const_expert_num, a_capacity, DTYPE_CODES[dtype], _p(ex), _p(idx),
                             _p(_c(topk_weights, np.float32)), _p(_c(assist_info, np.int32)),
                             _p(m), 0 if m is None else m.ndim, *[_p(a) for a in args],
                             comm_quant_mode, _p(out))
    return out


def combine_bwd(grad_out, expand_x, topk_weights, assist_info, *, k, a_capacity, dtype,
                mask=None, comm_quant_mode=0):
    """Returns (grad_expand (A, H), grad_w (BS, K) f32, abs_sum (BS, K) f64).

    Rows of grad_expand without a slot are left zero. With comm_quant_mode 2 the
    backward of the int8 round-trip combine: grad_w against the round-trip values,
    grad_expand straight through.
    """
    g = _c(grad_out, np.uint16)
    bs, h = g.shape
    ex = _c(expand_x, np.uint16)
    m = _c(mask, np.uint8)
    ge = np.zeros((a_capacity, h), np.uint16)
    gw = np.zeros((bs, k), np.float32)
    mag = np.zeros((bs, k), np.float64)
    fn = lib().oracle_combine_bwd_comm_quant if comm_quant_mode == 2 else lib().oracle_combine_bwd
    fn(bs, k, h, a_capacity, DTYPE_CODES[dtype], _p(g), _p(ex), _p(_c(topk_weights, np.float32)),
       _p(_c(assist_info, np.int32)), _p(m), 0 if m is None else m.ndim, _p(ge), _p(gw), _p(mag))
    return ge, gw, mag


def combine_bwd_special(grad_out, topk_idx, topk_weights, *, num_experts, dtype,
                        zero_expert_num=0, copy_expert_num=0, const_expert_num=0, mask=None,
                        ori_x=None, alpha1=None, alpha2=None, const_v=None):
    """Backward of the copy/const experts. Returns a dict with grad_w (BS, K; entries
    of other pairs are 0), abs_sum, grad_ori_x (BS, H) 16-bit, grad_alpha1/2, grad_v
    (Q, H) fp32 and their abs sums."""
    g = _c(grad_out, np.uint16)
    bs, h = g.shape
    idx = _c(topk_idx, np.int32)
    k = idx.shape[1]
    q = const_expert_num
    m = _c(mask, np.uint8)
    r = {"grad_w": np.zeros((bs, k), np.float32), "abs_sum": np.zeros((bs, k)),
         "grad_ori_x": np.zeros((bs, h), np.uint16)}
    for n in ("grad_alpha1", "grad_alpha2", "grad_v"):
        r[n] = np.zeros((q, h), np.float32)
    for n in ("abs_alpha1", "abs_alpha2", "abs_v"):
        r[n] = np.zeros((q, h))
    lib().oracle_combine_bwd_special(
        bs, k, h, num_experts, zero_expert_num, copy_expert_num, q, DTYPE_CODES[dtype], _p(g),
        _p(idx), _p(_c(topk_weights, np.float32)), _p(m), 0 if m is None else m.ndim,
        _p(_c(ori_x, np.uint16)), _p(_c(alpha1, np.uint16)), _p(_c(alpha2, np.uint16)),
        _p(_c(const_v, np.uint16)), _p(r["grad_w"]), _p(r["abs_sum"]), _p(r["grad_ori_x"]),
        _p(r["grad_alpha1"]), _p(r["grad_alpha2"]), _p(r["grad_v"]), _p(r["abs_alpha1"]),
        _p(r["abs_alpha2"]), _p(r["abs_v"]))
    return r


def dispatch_bwd(grad_in, assist_info, *, bs, k, a_capacity, dtype, mask=None):
    gi = _c(grad_in, np.uint16)
    h = gi.shape[1]
    m = _c(mask, np.uint8)
    gx = np.zeros((bs, h), np.uint16)
    lib().oracle_dispatch_bwd(bs, k, h, a_capacity, DTYPE_CODES[dtype], _p(gi),
                              _p(_c(assist_info, np.int32)), _p(m), 0 if m is None else m.ndim,
                              _p(gx))
    return gx


def run_chain(inputs: dict):
    """The whole path on one workload: layout -> permute -> expert stand-in ->
    combine fwd (-> combine bwd -> expert stand-in bwd -> dispatch bwd).

    Returns a dict of every intermediate and output.
    """
    import workloads

    wl = inputs["workload"]
    r: dict = {}
    r["counts"], r["send"], r["assist"], r["status"] = dispatch_layout(
        inputs["topk_idx"], wl.num_experts, wl.n_ids, wl.a_capacity, inputs["mask"])
    if wl.quant_mode == 2:
        r["expand_q"], r["scales"] = dispatch_permute_quant(
            inputs["x"], r["assist"], wl.k, wl.a_capacity, wl.dtype)
        r["y"] = workloads.expert_forward(inputs, r["expand_q"], r["scales"])
    else:
        r["expand_x"] = dispatch_permute(inputs["x"], r["assist"], wl.k, wl.a_capacity)
        r["y"] = workloads.expert_forward(inputs, r["expand_x"])
    r["out"] = combine_fwd(
        r["y"], inputs["topk_idx"], inputs["topk_weights"], r["assist"],
        num_experts=wl.num_experts, a_capacity=wl.a_capacity, dtype=wl.dtype,
        zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
        const_expert_num=wl.const_expert_num, mask=inputs["mask"], shared=inputs["shared"],
        ori_x=inputs["ori_x"], alpha1=inputs["alpha1"], alpha2=inputs["alpha2"],
        const_v=inputs["v"])
    if wl.backward:
        r["grad_expand"], r["grad_w"], r["abs_sum"] = combine_bwd(
            inputs["grad_out"], r["y"], inputs["topk_weights"], r["assist"], k=wl.k,
            a_capacity=wl.a_capacity, dtype=wl.dtype, mask=inputs["mask"])
        r["grad_in"] = workloads.expert_backward(inputs, r["grad_expand"])
        r["grad_x"] = dispatch_bwd(r["grad_in"], r["assist"], bs=wl.bs, k=wl.k,
                                   a_capacity=wl.a_capacity, dtype=wl.dtype, mask=inputs["mask"])
    return r
