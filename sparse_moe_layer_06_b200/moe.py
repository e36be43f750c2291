"""Thin Python binding of the C ABI in include/moe.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that the torch tensors it is handed are CUDA,
contiguous and of the expected dtype, passes their device pointers and the
current CUDA stream to the library, and raises if the library returns an error.
PyTorch only supplies device memory and streams.

The library is loaded from ``libmoe_b200.so`` next to this file; if it is
missing the first call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_BAD_INDEX = 4, 5, 6
MOE_F32, MOE_BF16 = 0, 1
(MOE_CALL_ROUTE, MOE_CALL_ROUTER_LOGITS, MOE_CALL_PERMUTE, MOE_CALL_FFN, MOE_CALL_COMBINE,
 MOE_CALL_FORWARD, MOE_CALL_ROUTER_STATS, MOE_CALL_FORWARD_FP8) = range(8)

EXPORTED = (
    "moe_workspace_size", "moe_status_string", "moe_router_logits", "moe_route", "moe_permute",
    "moe_grouped_swiglu_ffn", "moe_combine", "moe_forward", "moe_read_device_status",
    "moe_clear_device_status", "moe_launch_count", "moe_profile_start", "moe_profile_stop",
    "moe_route_noalloc", "moe_router_stats", "moe_quantize_weights_fp8", "moe_forward_fp8",
    "moe_check_wait_timeout",
)
ROUTE_NOALLOC_SCRATCH_BYTES = 1 << 20


class MoEProblemC(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("I", ctypes.c_int32), ("top_k", ctypes.c_int32), ("num_shared", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("clip_limit", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


class KernelTimeC(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_double)]


@dataclass(frozen=True)
class MoEProblem:
    T: int
    H: int
    E: int
    I: int
    top_k: int
    num_shared: int
    routed_scale: float
    clip_limit: float
    dtype: torch.dtype

    @classmethod
    def from_config(cls, cfg, T: int | None = None) -> "MoEProblem":
        return cls(T=cfg.T if T is None else T, H=cfg.H, E=cfg.E, I=cfg.I, top_k=cfg.top_k,
                   num_shared=cfg.num_shared, routed_scale=cfg.routed_scale,
                   clip_limit=cfg.clip_limit, dtype=cfg.dtype)

    def c(self) -> MoEProblemC:
        code = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}.get(self.dtype)
        if code is None:
            raise TypeError(f"unsupported dtype {self.dtype}")
        return MoEProblemC(self.T, self.H, self.E, self.I, self.top_k, self.num_shared,
                           self.routed_scale, self.clip_limit, code)


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmoe_b200.so (raises if it is not there: no fallback path exists)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m sparse_moe_layer_06_b200.build`; "
                "the MoE layer has no non-CUDA implementation")
        lib = ctypes.CDLL(path)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        PP = ctypes.POINTER(MoEProblemC)
        sig = {
            "moe_workspace_size": (SZ, [PP, I32]),
            "moe_status_string": (ctypes.c_char_p, [I32]),
            "moe_router_logits": (I32, [PP, P, P, P, P, SZ, P]),
            "moe_route": (I32, [PP, P, P, P, P, P, P, SZ, P]),
            "moe_permute": (I32, [PP, P, P, P, P, P, P, P, SZ, P]),
            "moe_grouped_swiglu_ffn": (I32, [PP, P, I64, P, I32, P, P, P, SZ, P]),
            "moe_combine": (I32, [PP, P, P, P, P, P, P, SZ, P]),
            "moe_forward": (I32, [PP, P, P, P, P, P, P, P, P, P, SZ, P]),
            "moe_read_device_status": (I32, [P, ctypes.POINTER(I32), P]),
            "moe_clear_device_status": (I32, [P, P]),
            "moe_launch_count": (I64, []),
            "moe_profile_start": (I32, [I32]),
            "moe_profile_stop": (I32, [ctypes.POINTER(KernelTimeC), I32, ctypes.POINTER(I32)]),
            "moe_route_noalloc": (I32, [PP, P, P, P, P, P, P]),
            "moe_router_stats": (I32, [PP, P, P, P, P, P, P, P, P, ctypes.c_float, P, SZ, P]),
            "moe_quantize_weights_fp8": (I32, [PP, I32, P, P, P, P, P]),
            "moe_forward_fp8": (I32, [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]),
            "moe_check_wait_timeout": (I32, [P, SZ, ctypes.POINTER(I32), P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, dtype=None, name="tensor", optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(status, what)


def moe_workspace_size(problem: MoEProblem, call: int) -> int:
    pc = problem.c()
    return int(load_library().moe_workspace_size(ctypes.byref(pc), call))


def alloc_workspace(problem: MoEProblem, call: int, device=None, extra: int = 0) -> torch.Tensor:
    """Caller-owned workspace (device bytes) for `call`; plumbing only."""
    n = moe_workspace_size(problem, call)
    if n == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_workspace_size")
    ws = torch.empty(n + extra, dtype=torch.uint8, device=device or "cuda")
    ws[:256].zero_()
    return ws


def moe_router_logits(problem, x, gate_w, logits, workspace, stream=None):
    pc = problem.c()
    _check(load_library().moe_router_logits(
        ctypes.byref(pc), _ptr(x, problem.dtype, "x"), _ptr(gate_w, problem.dtype, "gate_w"),
        _ptr(logits, torch.float32, "logits"), _ptr(workspace, None, "workspace"),
        workspace.numel(), _stream(stream)), "moe_router_logits")


def moe_route(problem, x, gate_w, logit_bias, topk_idx, topk_w, workspace, stream=None):
    pc = problem.c()
    _check(load_library().moe_route(
        ctypes.byref(pc), _ptr(x, problem.dtype, "x"), _ptr(gate_w, problem.dtype, "gate_w"),
        _ptr(logit_bias, torch.float32, "logit_bias", optional=True),
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)), "moe_route")


def moe_route_noalloc(problem, x, gate_w, logit_bias, topk_idx, topk_w, stream=None):
    """moe_route without a workspace: for callers that cannot allocate device
    memory (stream capture in progress, a framework allocator owning all
    memory, hot paths that must not synchronise).  Scratch is a fixed 1 MiB
    device array inside the library; T*E*4 + 256 bytes must fit in it.
    Calls that overlap on the GPU race on that array."""
    pc = problem.c()
    _check(load_library().moe_route_noalloc(
        ctypes.byref(pc), _ptr(x, problem.dtype, "x"), _ptr(gate_w, problem.dtype, "gate_w"),
        _ptr(logit_bias, torch.float32, "logit_bias", optional=True),
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
        _stream(stream)), "moe_route_noalloc")


def moe_router_stats(problem, x, gate_w, logit_bias, P_out, f_out, aux_out, ema_counts,
                     ema_total, momentum, workspace, stream=None):
    pc = problem.c()
    _check(load_library().moe_router_stats(
        ctypes.byref(pc), _ptr(x, problem.dtype, "x"), _ptr(gate_w, problem.dtype, "gate_w"),
        _ptr(logit_bias, torch.float32, "logit_bias", optional=True),
        _ptr(P_out, torch.float32, "P_out"), _ptr(f_out, torch.float32, "f_out"),
        _ptr(aux_out, torch.float32, "aux_out"),
        _ptr(ema_counts, torch.float32, "ema_counts", optional=True),
        _ptr(ema_total, torch.float32, "ema_total", optional=True), float(momentum),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)),
        "moe_router_stats")


def moe_quantize_weights_fp8(problem, w, q, scale_gu, scale_d, stream=None):
    """Encode [n,3,I,H] weights into E4M3 codes q (uint8, same shape) with
    scale_gu [n,2,I] and scale_d [n,H] (fp32); n is w.shape[0]."""
    pc = problem.c()
    _check(load_library().moe_quantize_weights_fp8(
        ctypes.byref(pc), int(w.shape[0]), _ptr(w, problem.dtype, "w"),
        _ptr(q, torch.uint8, "q"), _ptr(scale_gu, torch.float32, "scale_gu"),
        _ptr(scale_d, torch.float32, "scale_d"), _stream(stream)), "moe_quantize_weights_fp8")


def moe_forward_fp8(problem, x, gate_w, logit_bias, expert_q, expert_s_gu, expert_s_d,
                    shared_q, shared_s_gu, shared_s_d, out, topk_idx_out, topk_w_out, workspace,
                    stream=None):
    pc = problem.c()
    _check(load_library().moe_forward_fp8(
        ctypes.byref(pc), _ptr(x, torch.bfloat16, "x"), _ptr(gate_w, torch.bfloat16, "gate_w"),
        _ptr(logit_bias, torch.float32, "logit_bias", optional=True),
        _ptr(expert_q, torch.uint8, "expert_q"), _ptr(expert_s_gu, torch.float32, "expert_s_gu"),
        _ptr(expert_s_d, torch.float32, "expert_s_d"),
        _ptr(shared_q, torch.uint8, "shared_q", optional=True),
        _ptr(shared_s_gu, torch.float32, "shared_s_gu", optional=True),
        _ptr(shared_s_d, torch.float32, "shared_s_d", optional=True),
        _ptr(out, torch.bfloat16, "out"),
        _ptr(topk_idx_out, torch.int32, "topk_idx_out", optional=True),
        _ptr(topk_w_out, torch.float32, "topk_w_out", optional=True),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)), "moe_forward_fp8")


def moe_check_wait_timeout(workspace, stream=None) -> int:
    """Run the bounded-wait self-check; returns the bits of the waits that gave
    up (3 = both).  The workspace's error word is left at MOE_ERR_TIMEOUT."""
    out = ctypes.c_int32(0)
    _check(load_library().moe_check_wait_timeout(
        _ptr(workspace, None, "workspace"), workspace.numel(), ctypes.byref(out),
        _stream(stream)), "moe_check_wait_timeout")
    return int(out.value)


def moe_permute(problem, topk_idx, x, offsets, pos, src_token, x_perm, workspace, stream=None):
    pc = problem.c()
    _check(load_library().moe_permute(
        ctypes.byref(pc), _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(x, problem.dtype, "x"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(pos, torch.int32, "pos"),
        _ptr(src_token, torch.int32, "src_token"), _ptr(x_perm, problem.dtype, "x_perm"),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)), "moe_permute")


def moe_grouped_swiglu_ffn(problem, x_perm, offsets, n_groups, expert_w, y_perm, workspace,
                           stream=None):
    pc = problem.c()
    _check(load_library().moe_grouped_swiglu_ffn(
        ctypes.byref(pc), _ptr(x_perm, problem.dtype, "x_perm"), x_perm.shape[0],
        _ptr(offsets, torch.int32, "offsets"), int(n_groups),
        _ptr(expert_w, problem.dtype, "expert_w"), _ptr(y_perm, problem.dtype, "y_perm"),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)),
        "moe_grouped_swiglu_ffn")


def ffn_workspace_size(problem: MoEProblem, rows: int, n_groups: int) -> int:
    """Workspace bytes for moe_grouped_swiglu_ffn on `rows` rows in `n_groups` groups."""
    import dataclasses
    # the C sizing uses max(T*top_k, T) rows and E groups; express the request that way
    p = dataclasses.replace(problem, T=rows, top_k=1, E=max(1, n_groups))
    return moe_workspace_size(p, MOE_CALL_FFN)


def moe_combine(problem, y_perm, pos, topk_w, shared_y, out, workspace, stream=None):
    pc = problem.c()
    _check(load_library().moe_combine(
        ctypes.byref(pc), _ptr(y_perm, problem.dtype, "y_perm"), _ptr(pos, torch.int32, "pos"),
        _ptr(topk_w, torch.float32, "topk_w"),
        _ptr(shared_y, problem.dtype, "shared_y", optional=True), _ptr(out, problem.dtype, "out"),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)), "moe_combine")


def moe_forward(problem, x, gate_w, logit_bias, expert_w, shared_w, out, topk_idx_out,
                topk_w_out, workspace, stream=None):
    pc = problem.c()
    _check(load_library().moe_forward(
        ctypes.byref(pc), _ptr(x, problem.dtype, "x"), _ptr(gate_w, problem.dtype, "gate_w"),
        _ptr(logit_bias, torch.float32, "logit_bias", optional=True),
        _ptr(expert_w, problem.dtype, "expert_w"),
        _ptr(shared_w, problem.dtype, "shared_w", optional=True),
        _ptr(out, problem.dtype, "out"),
        _ptr(topk_idx_out, torch.int32, "topk_idx_out", optional=True),
        _ptr(topk_w_out, torch.float32, "topk_w_out", optional=True),
        _ptr(workspace, None, "workspace"), workspace.numel(), _stream(stream)), "moe_forward")


def moe_read_device_status(workspace, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(load_library().moe_read_device_status(_ptr(workspace, None, "workspace"),
                                                  ctypes.byref(out), _stream(stream)),
           "moe_read_device_status")
    return int(out.value)


def moe_clear_device_status(workspace, stream=None):
    _check(load_library().moe_clear_device_status(_ptr(workspace, None, "workspace"),
                                                   _stream(stream)), "moe_clear_device_status")


def moe_launch_count() -> int:
    return int(load_library().moe_launch_count())


def moe_profile_start(max_launches: int):
    _check(load_library().moe_profile_start(int(max_launches)), "moe_profile_start")


def moe_profile_stop(max_entries: int = 64) -> dict:
    arr = (KernelTimeC * max_entries)()
    n = ctypes.c_int32(0)
    _check(load_library().moe_profile_stop(arr, max_entries, ctypes.byref(n)), "moe_profile_stop")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms))
            for i in range(n.value)}
