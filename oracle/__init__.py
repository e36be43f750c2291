"""CPU oracle for the sparse MoE FFN layer forward -- TEST INFRASTRUCTURE.

This package is the plain, slow, fp64 reference that the CUDA path is checked
against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it; the product package never does, and the two
share no code.  All arithmetic lives in ``moe_oracle.c`` (plain C, double
precision, OpenMP over independent tokens or channels); this module only builds
that file with gcc and
marshals arguments through ctypes.

Inputs are torch CPU tensors in the stored dtype (``torch.bfloat16`` or
``torch.float32``); the C code widens every element exactly to double.
Outputs are float64 / int32 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_route.argtypes = [I64, I32, I32, I32, I32, P, P, P, D, P, I64, P, P, P, P]
            lib.oracle_forward.argtypes = [I64, I32, I32, I32, I32, I32, P, P, P, P, P, D, D,
                                           P, I64, P, P, P, P]
            lib.oracle_dense_bruteforce.argtypes = [I64, I32, I32, I32, I32, P, P, P, D, P, I64,
                                                    P, P]
            lib.oracle_expert_rows.argtypes = [I32, I32, I32, I32, P, P, P, D, P, P, I64, P]
            lib.oracle_permute.argtypes = [I64, I32, I32, P, P, P, P, P]
            lib.oracle_combine.argtypes = [I64, I32, I32, P, P, P, P, P]
            lib.oracle_router_stats.argtypes = [I64, I32, I32, I32, I32, P, P, P, D, P, P, P, P,
                                                P, P]
            lib.oracle_router_stats.restype = None
            lib.e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.e4m3_decode.restype = ctypes.c_double
            lib.e4m3_encode.argtypes = [ctypes.c_double]
            lib.e4m3_encode.restype = ctypes.c_uint8
            lib.pow2_scale.argtypes = [ctypes.c_double]
            lib.pow2_scale.restype = ctypes.c_double
            lib.oracle_quantize_weights_fp8.argtypes = [I32, I32, I32, I32, P, P, P, P]
            lib.oracle_quantize_weights_fp8.restype = None
            lib.oracle_forward_fp8.argtypes = [I64, I32, I32, I32, I32, I32, P, P, P, P, P, P, P,
                                               P, P, D, D, P, I64, P, P, P, P]
            lib.oracle_forward_fp8.restype = None
            lib.oracle_num_threads.restype = ctypes.c_int
            for f in (lib.oracle_route, lib.oracle_forward, lib.oracle_dense_bruteforce,
                      lib.oracle_expert_rows, lib.oracle_permute, lib.oracle_combine):
                f.restype = None
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _stored(t: torch.Tensor | None):
    """(keep-alive array, pointer, dtype code) for a stored input tensor."""
    if t is None:
        return None, None, None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        arr = t.view(torch.int16).numpy()
        return arr, arr.ctypes.data, BF16
    if t.dtype == torch.float32:
        arr = t.numpy()
        return arr, arr.ctypes.data, F32
    raise TypeError(f"oracle inputs must be bf16 or fp32, got {t.dtype}")


def _f32(t):
    if t is None:
        return None, None
    a = np.ascontiguousarray(t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else t,
                             dtype=np.float32)
    return a, a.ctypes.data


def _tokens(T: int, tokens):
    if tokens is None:
        tok = np.arange(T, dtype=np.int64)
    else:
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
        if tok.size and (tok.min() < 0 or tok.max() >= T):
            raise ValueError("token index out of range")
    return tok


def route(x, gate_w, top_k: int, scale: float, logit_bias=None, tokens=None):
    """Router steps 1-4 for the listed tokens (all tokens by default).

    Returns dict(logits [n,E] f64, probs [n,E] f64, idx [n,k] i32, w [n,k] f64).
    """
    T, H = x.shape
    E = gate_w.shape[0]
    xa, xp, dt = _stored(x)
    ga, gp, dt2 = _stored(gate_w)
    if dt != dt2:
        raise TypeError("x and gate_w must share a dtype")
    ba, bp = _f32(logit_bias)
    tok = _tokens(T, tokens)
    n = tok.size
    logits = np.zeros((n, E), np.float64)
    probs = np.zeros((n, E), np.float64)
    idx = np.zeros((n, top_k), np.int32)
    w = np.zeros((n, top_k), np.float64)
    if n:
        _load().oracle_route(T, H, E, top_k, dt, xp, gp, bp, float(scale), tok.ctypes.data, n,
                             logits.ctypes.data, probs.ctypes.data, idx.ctypes.data,
                             w.ctypes.data)
    return dict(logits=logits, probs=probs, idx=idx, w=w)


def forward(x, gate_w, expert_w, shared_w, top_k: int, scale: float, clip: float,
            logit_bias=None, tokens=None, forced_idx=None):
    """Full layer forward (steps 1-6) for the listed tokens.

    ``forced_idx`` ([n,k]) replaces the top-k sets; it must come from this
    oracle's own near-tie alternatives.  Returns dict(out [n,H], idx, w).
    """
    T, H = x.shape
    E, three, I, H2 = expert_w.shape
    assert three == 3 and H2 == H
    xa, xp, dt = _stored(x)
    ga, gp, _ = _stored(gate_w)
    ea, ep, _ = _stored(expert_w)
    sa, sp, _ = _stored(shared_w)
    ba, bp = _f32(logit_bias)
    tok = _tokens(T, tokens)
    n = tok.size
    fa = None
    fp = None
    if forced_idx is not None:
        fa = np.ascontiguousarray(np.asarray(forced_idx, dtype=np.int32).reshape(n, top_k))
        fp = fa.ctypes.data
    out = np.zeros((n, H), np.float64)
    idx = np.zeros((n, top_k), np.int32)
    w = np.zeros((n, top_k), np.float64)
    if n:
        _load().oracle_forward(T, H, E, top_k, I, dt, xp, gp, bp, ep, sp, float(scale),
                               float(clip), tok.ctypes.data, n, fp, out.ctypes.data,
                               idx.ctypes.data, w.ctypes.data)
    return dict(out=out, idx=idx, w=w)


def dense_bruteforce(x, expert_w, shared_w, dense_w, clip: float, tokens=None):
    """All-experts evaluation combined with a dense [n,E] weight matrix."""
    T, H = x.shape
    E, _, I, _ = expert_w.shape
    xa, xp, dt = _stored(x)
    ea, ep, _ = _stored(expert_w)
    sa, sp, _ = _stored(shared_w)
    tok = _tokens(T, tokens)
    n = tok.size
    dw = np.ascontiguousarray(np.asarray(dense_w, dtype=np.float64).reshape(n, E))
    out = np.zeros((n, H), np.float64)
    if n:
        _load().oracle_dense_bruteforce(T, H, E, I, dt, xp, ep, sp, float(clip),
                                        tok.ctypes.data, n, dw.ctypes.data, out.ctypes.data)
    return out


def expert_rows(x, expert_w, shared_w, row_token, row_expert, clip: float):
    """Per-row expert FFN output; row_expert == E selects the shared expert."""
    T, H = x.shape
    E, _, I, _ = expert_w.shape
    xa, xp, dt = _stored(x)
    ea, ep, _ = _stored(expert_w)
    sa, sp, _ = _stored(shared_w)
    rt = np.ascontiguousarray(np.asarray(row_token, dtype=np.int32))
    re = np.ascontiguousarray(np.asarray(row_expert, dtype=np.int32))
    if rt.size and (rt.min() < 0 or rt.max() >= T or re.min() < 0 or re.max() > E):
        raise ValueError("row token/expert out of range")
    if rt.size and re.max() == E and shared_w is None:
        raise ValueError("shared-expert rows need shared_w")
    out = np.zeros((rt.size, H), np.float64)
    if rt.size:
        _load().oracle_expert_rows(H, E, I, dt, xp, ep, sp, float(clip), rt.ctypes.data,
                                   re.ctypes.data, rt.size, out.ctypes.data)
    return out


def permute(idx, num_experts: int):
    """Dispatch bookkeeping: counts [E], offsets [E+1], pos [T,k], src [T*k]."""
    ia = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    T, k = ia.shape
    if ia.size and (ia.min() < 0 or ia.max() >= num_experts):
        raise ValueError("expert index out of range")
    counts = np.zeros(num_experts, np.int32)
    offsets = np.zeros(num_experts + 1, np.int32)
    pos = np.zeros((T, k), np.int32)
    src = np.zeros(T * k, np.int32)
    _load().oracle_permute(T, num_experts, k, ia.ctypes.data, counts.ctypes.data,
                           offsets.ctypes.data, pos.ctypes.data, src.ctypes.data)
    return dict(counts=counts, offsets=offsets, pos=pos, src=src)


def combine(y_perm, pos, w, shared_y=None):
    """out[t] = sum_j w[t,j] * y_perm[pos[t,j]] + shared_y[t] (float64)."""
    ya = np.ascontiguousarray(np.asarray(y_perm, dtype=np.float64))
    pa = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    wa = np.ascontiguousarray(np.asarray(w, dtype=np.float64))
    T, k = pa.shape
    H = ya.shape[1]
    sa = None
    sp = None
    if shared_y is not None:
        sa = np.ascontiguousarray(np.asarray(shared_y, dtype=np.float64))
        sp = sa.ctypes.data
    out = np.zeros((T, H), np.float64)
    _load().oracle_combine(T, H, k, ya.ctypes.data, pa.ctypes.data, wa.ctypes.data, sp,
                           out.ctypes.data)
    return out


def router_stats(x, gate_w, top_k: int, logit_bias=None, momentum: float = 0.9,
                 ema_counts=None, ema_total=None):
    """Load-balancing statistics over all tokens: dict(P [E], f [E], counts [E]
    int64, aux float, ema_counts [E] or None, ema_total float or None)."""
    T, H = x.shape
    E = gate_w.shape[0]
    xa, xp, dt = _stored(x)
    ga, gp, _ = _stored(gate_w)
    ba, bp = _f32(logit_bias)
    P = np.zeros(E, np.float64)
    f = np.zeros(E, np.float64)
    cnt = np.zeros(E, np.int64)
    aux = np.zeros(1, np.float64)
    ec = None if ema_counts is None else np.array(ema_counts, dtype=np.float64, copy=True)
    et = None if ema_total is None else np.array([ema_total], dtype=np.float64)
    _load().oracle_router_stats(T, H, E, top_k, dt, xp, gp, bp, float(momentum), P.ctypes.data,
                                f.ctypes.data, cnt.ctypes.data, aux.ctypes.data,
                                None if ec is None else ec.ctypes.data,
                                None if et is None else et.ctypes.data)
    return dict(P=P, f=f, counts=cnt, aux=float(aux[0]), ema_counts=ec,
                ema_total=None if et is None else float(et[0]))


def e4m3_decode(code: int) -> float:
    return float(_load().e4m3_decode(int(code) & 0xFF))


def e4m3_encode(v: float) -> int:
    return int(_load().e4m3_encode(float(v)))


def pow2_scale(amax: float) -> float:
    return float(_load().pow2_scale(float(amax)))


def quantize_weights_fp8(expert_w):
    """[E,3,I,H] weights -> (codes uint8 [E,3,I,H], gate/up row scales [E,2,I]
    f64, down column scales [E,H] f64)."""
    E, three, I, H = expert_w.shape
    wa, wp, dt = _stored(expert_w)
    q = np.zeros((E, 3, I, H), np.uint8)
    s_gu = np.zeros((E, 2, I), np.float64)
    s_d = np.zeros((E, H), np.float64)
    _load().oracle_quantize_weights_fp8(E, I, H, dt, wp, q.ctypes.data, s_gu.ctypes.data,
                                        s_d.ctypes.data)
    return q, s_gu, s_d


def forward_fp8(x, gate_w, q, s_gu, s_d, shared_q, shared_s_gu, shared_s_d, top_k: int,
                scale: float, clip: float, logit_bias=None, tokens=None, forced_idx=None):
    """Layer forward with FP8 expert weights (see moe_oracle.c).  q/s_gu/s_d as
    returned by quantize_weights_fp8; shared_* for one shared expert or None."""
    T, H = x.shape
    E = q.shape[0]
    I = q.shape[2]
    xa, xp, dt = _stored(x)
    ga, gp, _ = _stored(gate_w)
    ba, bp = _f32(logit_bias)
    qa = np.ascontiguousarray(q, dtype=np.uint8)
    sg = np.ascontiguousarray(s_gu, dtype=np.float64)
    sd = np.ascontiguousarray(s_d, dtype=np.float64)
    if shared_q is not None:
        sqa = np.ascontiguousarray(shared_q, dtype=np.uint8)
        ssg = np.ascontiguousarray(shared_s_gu, dtype=np.float64)
        ssd = np.ascontiguousarray(shared_s_d, dtype=np.float64)
        sq_p, ssg_p, ssd_p = sqa.ctypes.data, ssg.ctypes.data, ssd.ctypes.data
    else:
        sq_p = ssg_p = ssd_p = None
    tok = _tokens(T, tokens)
    n = tok.size
    fp = None
    if forced_idx is not None:
        fa = np.ascontiguousarray(np.asarray(forced_idx, dtype=np.int32).reshape(n, top_k))
        fp = fa.ctypes.data
    out = np.zeros((n, H), np.float64)
    idx = np.zeros((n, top_k), np.int32)
    w = np.zeros((n, top_k), np.float64)
    if n:
        _load().oracle_forward_fp8(T, H, E, top_k, I, dt, xp, gp, bp, qa.ctypes.data,
                                   sg.ctypes.data, sd.ctypes.data, sq_p, ssg_p, ssd_p,
                                   float(scale), float(clip), tok.ctypes.data, n, fp,
                                   out.ctypes.data, idx.ctypes.data, w.ctypes.data)
    return dict(out=out, idx=idx, w=w)


def near_tie_alternatives(probs_row: np.ndarray, k: int, rel: float = 1e-5):
    """Expert sets that are equally valid top-k choices at a near-tie.

    Given this oracle's probability vector for one token, returns the oracle's
    own top-k set first, then every set obtained by swapping selected experts
    whose probability lies within ``rel`` (relative) of the k-th largest for
    unselected ones within the same band.  Sets are returned as sorted tuples.
    """
    order = sorted(range(len(probs_row)), key=lambda e: (-probs_row[e], e))
    base = order[:k]
    pk = probs_row[order[k - 1]]
    band = [e for e in order if abs(probs_row[e] - pk) <= rel * pk]
    fixed = [e for e in base if e not in band]
    n_from_band = k - len(fixed)
    import itertools
    sets = [tuple(sorted(base))]
    for combo in itertools.combinations(band, n_from_band):
        s = tuple(sorted(fixed + list(combo)))
        if s not in sets:
            sets.append(s)
    return sets
