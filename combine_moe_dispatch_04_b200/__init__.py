"""Python binding of libmoe_dc.so, the B200 (sm_100a) MoE dispatch/combine library.

Argument marshalling only: every step runs in the library's CUDA kernels. PyTorch
supplies device memory and the current stream. The raw C entry points keep their C
names (``moe_dispatch_layout`` ...); the functions without the ``moe_`` prefix take
torch tensors, allocate outputs with torch, and raise ``MoeError`` on a non-OK status.

There is no CPU fallback: importing this package fails loudly when the library is
missing, and every call on a tensor that is not on a CUDA device raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_dc.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_ALIGN, MOE_ERR_CAPACITY, MOE_ERR_CUDA = range(6)
MOE_BF16, MOE_FP16 = 0, 1
MOE_DEV_BAD_ID, MOE_DEV_DUP_ID = 1, 2

# Every entry point include/moe_dc.h declares.
EXPORTS = ("moe_status_string", "moe_last_cuda_error", "moe_assist_info_elems",
           "moe_layout_workspace_bytes", "moe_dispatch_layout", "moe_dispatch_permute",
           "moe_combine_fwd", "moe_combine_bwd", "moe_dispatch_bwd",
           "moe_dispatch_layout_noalloc", "moe_layout_noalloc_max_workspace_bytes",
           "moe_combine_fwd_comm_quant", "moe_dispatch", "moe_combine_bwd_special",
           "moe_combine_bwd_special_workspace_bytes", "moe_dispatch_permute_smooth",
           "moe_async_wait_timeouts", "moe_combine_fwd_comm_quant_ws",
           "moe_combine_fwd_comm_quant_workspace_bytes", "moe_combine_bwd_comm_quant",
           "moe_test_combine_fwd_comm_quant_wait_timeout",
           "moe_test_dispatch_permute_smooth_wait_timeout")


class MoeShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "bs", "k", "h", "num_experts", "zero_expert_num", "copy_expert_num",
        "const_expert_num", "a_capacity", "dtype", "mask_ndim")]


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            msg += f" (cudaError {_lib.moe_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python combine_moe_dispatch_04_b200/build.py`"
            " (there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(MoeShape)
    L.moe_status_string.argtypes, L.moe_status_string.restype = [I], ctypes.c_char_p
    L.moe_last_cuda_error.argtypes, L.moe_last_cuda_error.restype = [], I
    L.moe_assist_info_elems.argtypes, L.moe_assist_info_elems.restype = [S], ctypes.c_size_t
    L.moe_layout_workspace_bytes.argtypes = [S]
    L.moe_layout_workspace_bytes.restype = ctypes.c_size_t
    L.moe_dispatch_layout.argtypes = [S, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_dispatch_permute.argtypes = [S, P, P, P, I, P, P, P]
    L.moe_dispatch_permute_smooth.argtypes = [S, P, P, P, P, P, P, P, P]
    L.moe_async_wait_timeouts.argtypes, L.moe_async_wait_timeouts.restype = [], ctypes.c_uint32
    L.moe_combine_fwd.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P]
    L.moe_combine_fwd_comm_quant.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, I, P, P]
    L.moe_combine_fwd_comm_quant_ws.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, I, P, P,
                                                ctypes.c_size_t, P]
    L.moe_combine_fwd_comm_quant_workspace_bytes.argtypes = [S]
    L.moe_combine_fwd_comm_quant_workspace_bytes.restype = ctypes.c_size_t
    L.moe_dispatch.argtypes = [S, P, P, P, I, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_combine_bwd_special.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                          ctypes.c_size_t, P]
    L.moe_combine_bwd_special_workspace_bytes.argtypes = [S]
    L.moe_combine_bwd_special_workspace_bytes.restype = ctypes.c_size_t
    L.moe_combine_bwd.argtypes = [S, P, P, P, P, P, P, P, P, P]
    L.moe_combine_bwd_comm_quant.argtypes = [S, P, P, P, P, P, P, I, P, P, P]
    U64 = ctypes.c_uint64
    L.moe_test_combine_fwd_comm_quant_wait_timeout.argtypes = [S, P, P, P, P, P, P, P, P, P, P,
                                                               P, U64, I, P]
    L.moe_test_dispatch_permute_smooth_wait_timeout.argtypes = [S, P, P, P, P, P, P, P, U64, I,
                                                                P]
    L.moe_dispatch_bwd.argtypes = [S, P, P, P, P, P]
    L.moe_dispatch_layout_noalloc.argtypes = [S, P, P, P, P, P, P, P]
    L.moe_layout_noalloc_max_workspace_bytes.argtypes = []
    L.moe_layout_noalloc_max_workspace_bytes.restype = ctypes.c_size_t
    for n in ("moe_dispatch_layout", "moe_dispatch_permute", "moe_combine_fwd",
              "moe_combine_bwd", "moe_dispatch_bwd", "moe_dispatch_layout_noalloc",
              "moe_combine_fwd_comm_quant", "moe_dispatch", "moe_combine_bwd_special",
              "moe_dispatch_permute_smooth", "moe_combine_fwd_comm_quant_ws",
              "moe_combine_bwd_comm_quant", "moe_test_combine_fwd_comm_quant_wait_timeout",
              "moe_test_dispatch_permute_smooth_wait_timeout"):
        getattr(L, n).restype = I
    return L


_lib = _load()

# Raw C entry points, same names as the header.
moe_status_string = _lib.moe_status_string
moe_last_cuda_error = _lib.moe_last_cuda_error
moe_assist_info_elems = _lib.moe_assist_info_elems
moe_layout_workspace_bytes = _lib.moe_layout_workspace_bytes
moe_dispatch_layout = _lib.moe_dispatch_layout
moe_dispatch_permute = _lib.moe_dispatch_permute
moe_dispatch_permute_smooth = _lib.moe_dispatch_permute_smooth
moe_async_wait_timeouts = _lib.moe_async_wait_timeouts
moe_combine_fwd = _lib.moe_combine_fwd
moe_combine_bwd = _lib.moe_combine_bwd
moe_combine_bwd_comm_quant = _lib.moe_combine_bwd_comm_quant
moe_test_combine_fwd_comm_quant_wait_timeout = _lib.moe_test_combine_fwd_comm_quant_wait_timeout
moe_test_dispatch_permute_smooth_wait_timeout = (
    _lib.moe_test_dispatch_permute_smooth_wait_timeout)
moe_dispatch_bwd = _lib.moe_dispatch_bwd
moe_dispatch_layout_noalloc = _lib.moe_dispatch_layout_noalloc
moe_combine_fwd_comm_quant = _lib.moe_combine_fwd_comm_quant
moe_combine_fwd_comm_quant_ws = _lib.moe_combine_fwd_comm_quant_ws
moe_combine_fwd_comm_quant_workspace_bytes = _lib.moe_combine_fwd_comm_quant_workspace_bytes
moe_dispatch = _lib.moe_dispatch
moe_combine_bwd_special = _lib.moe_combine_bwd_special
moe_combine_bwd_special_workspace_bytes = _lib.moe_combine_bwd_special_workspace_bytes
moe_layout_noalloc_max_workspace_bytes = _lib.moe_layout_noalloc_max_workspace_bytes


def library():
    """The loaded ctypes library."""
    return _lib


@dataclass(frozen=True)
class Shape:
    bs: int
    k: int
    h: int
    num_experts: int
    zero_expert_num: int = 0
    copy_expert_num: int = 0
    const_expert_num: int = 0
    a_capacity: int = 0  # 0: BS * K
    dtype: int = MOE_BF16
    mask_ndim: int = 0

    def c(self) -> MoeShape:
        return MoeShape(self.bs, self.k, self.h, self.num_experts, self.zero_expert_num,
                        self.copy_expert_num, self.const_expert_num,
                        self.a_capacity or self.bs * self.k, self.dtype, self.mask_ndim)

    @property
    def A(self) -> int:
        return self.a_capacity or self.bs * self.k

    @property
    def n_ids(self) -> int:
        return (self.num_experts + self.zero_expert_num + self.copy_expert_num
                + self.const_expert_num)


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoeError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor is not on a CUDA device (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _torch_dtype(shape: Shape):
    import torch

    return torch.bfloat16 if shape.dtype == MOE_BF16 else torch.float16


@dataclass
class Layout:
    expert_token_nums: object  # int32 (E,)
    ep_send_counts: object     # int32 (E + 1,)
    assist_info: object        # int32 (A + BS*K,)
    dev_status: object         # uint32-as-int32 (1,)


def layout_workspace(shape: Shape, device=None):
    """Workspace tensor for dispatch_layout (None when none is needed)."""
    import torch

    n = moe_layout_workspace_bytes(ctypes.byref(shape.c()))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda") if n else None


def dispatch_layout(shape: Shape, topk_idx, x_active_mask=None, *, workspace=None, out=None,
                    stream=None) -> Layout:
    import torch

    dev = topk_idx.device
    if out is None:
        out = Layout(torch.empty(shape.num_experts, dtype=torch.int32, device=dev),
                     torch.empty(shape.num_experts + 1, dtype=torch.int32, device=dev),
                     torch.empty(shape.A + shape.bs * shape.k, dtype=torch.int32, device=dev),
                     torch.empty(1, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = layout_workspace(shape, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_dispatch_layout", moe_dispatch_layout(
        ctypes.byref(shape.c()), _ptr(topk_idx), _ptr(x_active_mask), _ptr(out.expert_token_nums),
        _ptr(out.ep_send_counts), _ptr(out.assist_info), _ptr(out.dev_status), _ptr(workspace),
        ws_bytes, _stream(stream)))
    return out


def dispatch_layout_noalloc(shape: Shape, topk_idx, x_active_mask=None, *, out: Layout,
                            stream=None) -> Layout:
    """The layout without a workspace, for callers that cannot allocate device memory:
    the library's own fixed scratch array stands in for it. ``out`` (caller-provided
    outputs) is required, since this path allocates nothing."""
    _check("moe_dispatch_layout_noalloc", moe_dispatch_layout_noalloc(
        ctypes.byref(shape.c()), _ptr(topk_idx), _ptr(x_active_mask), _ptr(out.expert_token_nums),
        _ptr(out.ep_send_counts), _ptr(out.assist_info), _ptr(out.dev_status), _stream(stream)))
    return out


def dispatch(shape: Shape, topk_idx, x, x_active_mask=None, comm_quant_mode: int = 0, *,
             workspace=None, layout: Layout | None = None, expand_x=None, dynamic_scales=None,
             stream=None):
    """Layout and permute in one call (one launch for BS <= 1024 without quantisation).
    Returns (layout, expand_x, dynamic_scales)."""
    import torch

    dev = topk_idx.device
    if layout is None:
        layout = Layout(torch.empty(shape.num_experts, dtype=torch.int32, device=dev),
                        torch.empty(shape.num_experts + 1, dtype=torch.int32, device=dev),
                        torch.empty(shape.A + shape.bs * shape.k, dtype=torch.int32, device=dev),
                        torch.empty(1, dtype=torch.int32, device=dev))
    if expand_x is None:
        dt = torch.int8 if comm_quant_mode == 2 else _torch_dtype(shape)
        expand_x = torch.empty(shape.A, shape.h, dtype=dt, device=dev)
    if comm_quant_mode == 2 and dynamic_scales is None:
        dynamic_scales = torch.empty(shape.A, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = layout_workspace(shape, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_dispatch", moe_dispatch(
        ctypes.byref(shape.c()), _ptr(topk_idx), _ptr(x_active_mask), _ptr(x), comm_quant_mode,
        _ptr(layout.expert_token_nums), _ptr(layout.ep_send_counts), _ptr(layout.assist_info),
        _ptr(layout.dev_status), _ptr(expand_x), _ptr(dynamic_scales), _ptr(workspace), ws_bytes,
        _stream(stream)))
    return layout, expand_x, dynamic_scales


def dispatch_permute(shape: Shape, x, layout: Layout, comm_quant_mode: int = 0, *,
                     expand_x=None, dynamic_scales=None, stream=None):
    """Returns expand_x (A, H) (int8 under comm_quant_mode 2) and dynamic_scales (or None)."""
    import torch

    if expand_x is None:
        dt = torch.int8 if comm_quant_mode == 2 else _torch_dtype(shape)
        expand_x = torch.empty(shape.A, shape.h, dtype=dt, device=x.device)
    if comm_quant_mode == 2 and dynamic_scales is None:
        dynamic_scales = torch.empty(shape.A, dtype=torch.float32, device=x.device)
    _check("moe_dispatch_permute", moe_dispatch_permute(
        ctypes.byref(shape.c()), _ptr(x), _ptr(layout.assist_info), _ptr(layout.ep_send_counts),
        comm_quant_mode, _ptr(expand_x), _ptr(dynamic_scales), _stream(stream)))
    return expand_x, dynamic_scales


def dispatch_permute_smooth(shape: Shape, x, topk_idx, layout: Layout, smooth_scales, *,
                            expand_x=None, dynamic_scales=None, stream=None):
    """int8 dispatch of x[t] * smooth_scales[e] per slot: (expand_x (A, H) int8, scales (A,))."""
    import torch

    if expand_x is None:
        expand_x = torch.empty(shape.A, shape.h, dtype=torch.int8, device=x.device)
    if dynamic_scales is None:
        dynamic_scales = torch.empty(shape.A, dtype=torch.float32, device=x.device)
    _check("moe_dispatch_permute_smooth", moe_dispatch_permute_smooth(
        ctypes.byref(shape.c()), _ptr(x), _ptr(topk_idx), _ptr(layout.assist_info),
        _ptr(layout.ep_send_counts), _ptr(smooth_scales), _ptr(expand_x), _ptr(dynamic_scales),
        _stream(stream)))
    return expand_x, dynamic_scales


def combine_fwd(shape: Shape, expand_x, topk_idx, topk_weights, layout: Layout, *,
                x_active_mask=None, shared_expert_x=None, ori_x=None, const_alpha_1=None,
                const_alpha_2=None, const_v=None, comm_quant_mode=0, workspace=None,
                use_workspace=True, out=None, stream=None):
    """Combine forward. With comm_quant_mode 2, a workspace (allocated here unless
    given, or none with use_workspace=False) lets shapes without zero/copy/const
    experts take the two-pass kernels; the result is the same either way."""
    import torch

    if out is None:
        out = torch.empty(shape.bs, shape.h, dtype=_torch_dtype(shape), device=expand_x.device)
    args = (ctypes.byref(shape.c()), _ptr(expand_x), _ptr(topk_idx), _ptr(topk_weights),
            _ptr(layout.assist_info), _ptr(layout.ep_send_counts), _ptr(x_active_mask),
            _ptr(shared_expert_x), _ptr(ori_x), _ptr(const_alpha_1), _ptr(const_alpha_2),
            _ptr(const_v))
    if comm_quant_mode == 0:
        _check("moe_combine_fwd", moe_combine_fwd(*args, _ptr(out), _stream(stream)))
        return out
    nbytes = 0
    if use_workspace:
        nbytes = moe_combine_fwd_comm_quant_workspace_bytes(ctypes.byref(shape.c()))
        if workspace is None and nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=expand_x.device)
    else:
        workspace = None
    _check("moe_combine_fwd_comm_quant_ws", moe_combine_fwd_comm_quant_ws(
        *args, comm_quant_mode, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream(stream)))
    return out


def combine_bwd(shape: Shape, grad_out, expand_x, topk_weights, layout: Layout, *,
                topk_idx=None, x_active_mask=None, comm_quant_mode=0, grad_expand=None,
                grad_w=None, stream=None):
    """Returns (grad_expand (A, H), grad_w (BS, K) fp32). Rows without a slot are not
    written. comm_quant_mode 2: the backward of the int8 round-trip combine."""
    import torch

    if grad_expand is None:
        grad_expand = torch.empty(shape.A, shape.h, dtype=_torch_dtype(shape),
                                  device=grad_out.device)
    if grad_w is None:
        grad_w = torch.empty(shape.bs, shape.k, dtype=torch.float32, device=grad_out.device)
    _check("moe_combine_bwd_comm_quant", moe_combine_bwd_comm_quant(
        ctypes.byref(shape.c()), _ptr(grad_out), _ptr(expand_x), _ptr(topk_idx),
        _ptr(topk_weights), _ptr(layout.assist_info), _ptr(x_active_mask), comm_quant_mode,
        _ptr(grad_expand), _ptr(grad_w), _stream(stream)))
    return grad_expand, grad_w


def combine_bwd_special(shape: Shape, grad_out, topk_idx, topk_weights, ori_x, *,
                        x_active_mask=None, const_alpha_1=None, const_alpha_2=None,
                        const_v=None, grad_w=None, workspace=None, out=None, stream=None):
    """Backward of the copy/const experts. Fills the copy/const entries of grad_w (a new
    zero tensor when None) and returns (grad_w, grad_ori_x, grad_alpha_1, grad_alpha_2,
    grad_v); the last three are None without const experts. `out` may hold the last
    four tensors, preallocated."""
    import torch

    dev = grad_out.device
    if grad_w is None:
        grad_w = torch.zeros(shape.bs, shape.k, dtype=torch.float32, device=dev)
    if out is not None:
        grad_ori, ga1, ga2, gv = out
    else:
        grad_ori = torch.empty(shape.bs, shape.h, dtype=_torch_dtype(shape), device=dev)
        ga1 = ga2 = gv = None
        if shape.const_expert_num:
            ga1, ga2, gv = (torch.empty(shape.const_expert_num, shape.h, dtype=torch.float32,
                                        device=dev) for _ in range(3))
    if workspace is None:
        n = moe_combine_bwd_special_workspace_bytes(ctypes.byref(shape.c()))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=dev) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_combine_bwd_special", moe_combine_bwd_special(
        ctypes.byref(shape.c()), _ptr(grad_out), _ptr(topk_idx), _ptr(topk_weights),
        _ptr(x_active_mask), _ptr(ori_x), _ptr(const_alpha_1), _ptr(const_alpha_2),
        _ptr(const_v), _ptr(grad_w), _ptr(grad_ori), _ptr(ga1), _ptr(ga2), _ptr(gv),
        _ptr(workspace), ws_bytes, _stream(stream)))
    return grad_w, grad_ori, ga1, ga2, gv


def dispatch_bwd(shape: Shape, grad_expand_in, layout: Layout, *, x_active_mask=None,
                 grad_x=None, stream=None):
    import torch

    if grad_x is None:
        grad_x = torch.empty(shape.bs, shape.h, dtype=_torch_dtype(shape),
                             device=grad_expand_in.device)
    _check("moe_dispatch_bwd", moe_dispatch_bwd(
        ctypes.byref(shape.c()), _ptr(grad_expand_in), _ptr(layout.assist_info),
        _ptr(x_active_mask), _ptr(grad_x), _stream(stream)))
    return grad_x
