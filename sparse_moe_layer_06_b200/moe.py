"""Thin Python binding of the C ABI in include/moe.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that the torch tensors it is handed are CUDA,
contiguous, of the expected dtype and at least as large as the problem needs
(the kernels take their extents from the problem, so a short tensor would be
accessed out of bounds on the device), passes their device pointers and the
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
    "moe_check_wait_timeout", "moe_expert_tile_rows",
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
            "moe_expert_tile_rows": (I32, [PP, ctypes.POINTER(I32), ctypes.POINTER(I32)]),
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


def _ptr(t, dtype=None, name="tensor", optional=False, numel=None):
    """Device pointer of `t` after checking it: a contiguous CUDA tensor of
    `dtype` holding at least `numel` elements (the kernels take their extents
    from the problem, not from the tensor, so a short tensor would be read or
    written out of bounds on the device)."""
    return _ptrs((t, dtype, name, optional, numel))[0]


def _ptrs(*specs):
    """Pointers of several operands, each spec (tensor, dtype, name, optional,
    numel).  Every operand's type, dtype, size and layout is checked before
    any operand's device, so the first error names the operand that is
    actually wrong."""
    for t, dtype, name, optional, numel in specs:
        if t is None:
            if optional:
                continue
            raise ValueError(f"{name} is required")
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a CUDA tensor")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if numel is not None and t.numel() < numel:
            raise ValueError(f"{name} has {t.numel()} elements, the problem needs {numel}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    out = []
    for t, _, name, _, _ in specs:
        if t is None:
            out.append(None)
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        out.append(ctypes.c_void_p(t.data_ptr()))
    return out


def _spec(t, dtype=None, name="tensor", optional=False, numel=None):
    return (t, dtype, name, optional, numel)


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


def _ws(workspace):
    return _spec(workspace, None, "workspace")


def moe_router_logits(problem, x, gate_w, logits, workspace, stream=None):
    pc = problem.c()
    T, H, E = problem.T, problem.H, problem.E
    ptrs = _ptrs(_spec(x, problem.dtype, "x", numel=T * H),
                 _spec(gate_w, problem.dtype, "gate_w", numel=E * H),
                 _spec(logits, torch.float32, "logits", numel=T * E), _ws(workspace))
    _check(load_library().moe_router_logits(ctypes.byref(pc), *ptrs, workspace.numel(),
                                            _stream(stream)), "moe_router_logits")


def _route_specs(problem, x, gate_w, logit_bias, topk_idx, topk_w):
    T, H, E, k = problem.T, problem.H, problem.E, problem.top_k
    return (_spec(x, problem.dtype, "x", numel=T * H),
            _spec(gate_w, problem.dtype, "gate_w", numel=E * H),
            _spec(logit_bias, torch.float32, "logit_bias", optional=True, numel=E),
            _spec(topk_idx, torch.int32, "topk_idx", numel=T * k),
            _spec(topk_w, torch.float32, "topk_w", numel=T * k))


def moe_route(problem, x, gate_w, logit_bias, topk_idx, topk_w, workspace, stream=None):
    pc = problem.c()
    ptrs = _ptrs(*_route_specs(problem, x, gate_w, logit_bias, topk_idx, topk_w), _ws(workspace))
    _check(load_library().moe_route(ctypes.byref(pc), *ptrs, workspace.numel(), _stream(stream)),
           "moe_route")


def moe_route_noalloc(problem, x, gate_w, logit_bias, topk_idx, topk_w, stream=None):
    """moe_route without a workspace: for callers that cannot allocate device
    memory (stream capture in progress, a framework allocator owning all
    memory, hot paths that must not synchronise).  Scratch is a fixed 1 MiB
    device array inside the library; T*E*4 + 256 bytes must fit in it.
    Calls that overlap on the GPU race on that array."""
    pc = problem.c()
    ptrs = _ptrs(*_route_specs(problem, x, gate_w, logit_bias, topk_idx, topk_w))
    _check(load_library().moe_route_noalloc(ctypes.byref(pc), *ptrs, _stream(stream)),
           "moe_route_noalloc")


def moe_router_stats(problem, x, gate_w, logit_bias, P_out, f_out, aux_out, ema_counts,
                     ema_total, momentum, workspace, stream=None):
    pc = problem.c()
    T, H, E = problem.T, problem.H, problem.E
    ptrs = _ptrs(_spec(x, problem.dtype, "x", numel=T * H),
                 _spec(gate_w, problem.dtype, "gate_w", numel=E * H),
                 _spec(logit_bias, torch.float32, "logit_bias", optional=True, numel=E),
                 _spec(P_out, torch.float32, "P_out", numel=E),
                 _spec(f_out, torch.float32, "f_out", numel=E),
                 _spec(aux_out, torch.float32, "aux_out", numel=1),
                 _spec(ema_counts, torch.float32, "ema_counts", optional=True, numel=E),
                 _spec(ema_total, torch.float32, "ema_total", optional=True, numel=1),
                 _ws(workspace))
    _check(load_library().moe_router_stats(ctypes.byref(pc), *ptrs[:8], float(momentum),
                                           ptrs[8], workspace.numel(), _stream(stream)),
           "moe_router_stats")


def moe_quantize_weights_fp8(problem, w, q, scale_gu, scale_d, stream=None):
    """Encode [n,3,I,H] weights into E4M3 codes q (uint8, same shape) with
    scale_gu [n,2,I] and scale_d [n,H] (fp32); n is w.shape[0]."""
    pc = problem.c()
    n, H, I = int(w.shape[0]), problem.H, problem.I
    ptrs = _ptrs(_spec(w, problem.dtype, "w", numel=n * 3 * I * H),
                 _spec(q, torch.uint8, "q", numel=n * 3 * I * H),
                 _spec(scale_gu, torch.float32, "scale_gu", numel=n * 2 * I),
                 _spec(scale_d, torch.float32, "scale_d", numel=n * H))
    _check(load_library().moe_quantize_weights_fp8(ctypes.byref(pc), n, *ptrs, _stream(stream)),
           "moe_quantize_weights_fp8")


def moe_forward_fp8(problem, x, gate_w, logit_bias, expert_q, expert_s_gu, expert_s_d,
                    shared_q, shared_s_gu, shared_s_d, out, topk_idx_out, topk_w_out, workspace,
                    stream=None):
    pc = problem.c()
    T, H, E, I, k = problem.T, problem.H, problem.E, problem.I, problem.top_k
    ptrs = _ptrs(_spec(x, torch.bfloat16, "x", numel=T * H),
                 _spec(gate_w, torch.bfloat16, "gate_w", numel=E * H),
                 _spec(logit_bias, torch.float32, "logit_bias", optional=True, numel=E),
                 _spec(expert_q, torch.uint8, "expert_q", numel=E * 3 * I * H),
                 _spec(expert_s_gu, torch.float32, "expert_s_gu", numel=E * 2 * I),
                 _spec(expert_s_d, torch.float32, "expert_s_d", numel=E * H),
                 _spec(shared_q, torch.uint8, "shared_q", optional=True, numel=3 * I * H),
                 _spec(shared_s_gu, torch.float32, "shared_s_gu", optional=True, numel=2 * I),
                 _spec(shared_s_d, torch.float32, "shared_s_d", optional=True, numel=H),
                 _spec(out, torch.bfloat16, "out", numel=T * H),
                 _spec(topk_idx_out, torch.int32, "topk_idx_out", optional=True, numel=T * k),
                 _spec(topk_w_out, torch.float32, "topk_w_out", optional=True, numel=T * k),
                 _ws(workspace))
    _check(load_library().moe_forward_fp8(ctypes.byref(pc), *ptrs, workspace.numel(),
                                          _stream(stream)), "moe_forward_fp8")


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
    T, H, E, k = problem.T, problem.H, problem.E, problem.top_k
    ptrs = _ptrs(_spec(topk_idx, torch.int32, "topk_idx", numel=T * k),
                 _spec(x, problem.dtype, "x", numel=T * H),
                 _spec(offsets, torch.int32, "offsets", numel=E + 1),
                 _spec(pos, torch.int32, "pos", numel=T * k),
                 _spec(src_token, torch.int32, "src_token", numel=T * k),
                 _spec(x_perm, problem.dtype, "x_perm", numel=T * k * H), _ws(workspace))
    _check(load_library().moe_permute(ctypes.byref(pc), *ptrs, workspace.numel(),
                                      _stream(stream)), "moe_permute")


def moe_grouped_swiglu_ffn(problem, x_perm, offsets, n_groups, expert_w, y_perm, workspace,
                           stream=None):
    pc = problem.c()
    H, I, g = problem.H, problem.I, int(n_groups)
    if not isinstance(x_perm, torch.Tensor) or x_perm.dim() != 2 or x_perm.shape[1] != H:
        raise ValueError(f"x_perm must be a [rows, {H}] tensor")
    rows = int(x_perm.shape[0])
    ptrs = _ptrs(_spec(x_perm, problem.dtype, "x_perm"),
                 _spec(offsets, torch.int32, "offsets", numel=max(0, g) + 1),
                 _spec(expert_w, problem.dtype, "expert_w", numel=max(0, g) * 3 * I * H),
                 _spec(y_perm, problem.dtype, "y_perm", numel=rows * H), _ws(workspace))
    x_p, off_p, w_p, y_p, ws_p = ptrs
    _check(load_library().moe_grouped_swiglu_ffn(ctypes.byref(pc), x_p, rows, off_p, g, w_p, y_p,
                                                 ws_p, workspace.numel(), _stream(stream)),
           "moe_grouped_swiglu_ffn")


def ffn_workspace_size(problem: MoEProblem, rows: int, n_groups: int) -> int:
    """Workspace bytes for moe_grouped_swiglu_ffn on `rows` rows in `n_groups` groups."""
    import dataclasses
    # the C sizing uses max(T*top_k, T) rows and E groups; express the request that way
    p = dataclasses.replace(problem, T=rows, top_k=1, E=max(1, n_groups))
    return moe_workspace_size(p, MOE_CALL_FFN)


def moe_combine(problem, y_perm, pos, topk_w, shared_y, out, workspace, stream=None):
    pc = problem.c()
    T, H, k = problem.T, problem.H, problem.top_k
    ptrs = _ptrs(_spec(y_perm, problem.dtype, "y_perm", numel=T * k * H),
                 _spec(pos, torch.int32, "pos", numel=T * k),
                 _spec(topk_w, torch.float32, "topk_w", numel=T * k),
                 _spec(shared_y, problem.dtype, "shared_y", optional=True, numel=T * H),
                 _spec(out, problem.dtype, "out", numel=T * H), _ws(workspace))
    _check(load_library().moe_combine(ctypes.byref(pc), *ptrs, workspace.numel(),
                                      _stream(stream)), "moe_combine")


def moe_forward(problem, x, gate_w, logit_bias, expert_w, shared_w, out, topk_idx_out,
                topk_w_out, workspace, stream=None):
    pc = problem.c()
    T, H, E, I, k = problem.T, problem.H, problem.E, problem.I, problem.top_k
    ptrs = _ptrs(_spec(x, problem.dtype, "x", numel=T * H),
                 _spec(gate_w, problem.dtype, "gate_w", numel=E * H),
                 _spec(logit_bias, torch.float32, "logit_bias", optional=True, numel=E),
                 _spec(expert_w, problem.dtype, "expert_w", numel=E * 3 * I * H),
                 _spec(shared_w, problem.dtype, "shared_w", optional=True, numel=3 * I * H),
                 _spec(out, problem.dtype, "out", numel=T * H),
                 _spec(topk_idx_out, torch.int32, "topk_idx_out", optional=True, numel=T * k),
                 _spec(topk_w_out, torch.float32, "topk_w_out", optional=True, numel=T * k),
                 _ws(workspace))
    _check(load_library().moe_forward(ctypes.byref(pc), *ptrs, workspace.numel(),
                                      _stream(stream)), "moe_forward")


def moe_expert_tile_rows(problem) -> tuple[int, int]:
    """(gate/up, down) token-row tile widths of the expert GEMMs for `problem`."""
    pc = problem.c()
    gu, dn = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load_library().moe_expert_tile_rows(ctypes.byref(pc), ctypes.byref(gu),
                                                ctypes.byref(dn)), "moe_expert_tile_rows")
    return int(gu.value), int(dn.value)


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
