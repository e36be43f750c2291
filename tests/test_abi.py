"""CPU checks of the C-ABI library: it builds, loads, exports every entry point
declared in include/moe.h, and its host-side validation rejects bad calls
before touching the GPU (no CUDA call is made by anything tested here)."""
import ctypes
import os
import re

import pytest
import torch

from sparse_moe_layer_06_b200 import build, moe
from sparse_moe_layer_06_b200.workloads import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def header_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_functions()
    for required in ("moe_route", "moe_permute", "moe_grouped_swiglu_ffn", "moe_combine",
                     "moe_forward", "moe_workspace_size", "moe_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert set(names) == set(moe.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_library_is_sm100a_only_build(lib):
    # the build flags target exactly sm_100a
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)
    assert os.path.getsize(build.LIB) > 0


def test_status_strings(lib):
    assert moe.status_string(0) == "ok"
    assert "workspace" in moe.status_string(3)
    assert moe.status_string(99) == "unknown status"


def problem(**kw):
    base = dict(T=128, H=256, E=16, I=128, top_k=2, num_shared=1, routed_scale=2.827,
                clip_limit=10.0, dtype=torch.bfloat16)
    base.update(kw)
    return moe.MoEProblem(**base)


def test_workspace_sizes_monotone_and_validated(lib):
    p = problem()
    sizes = {c: moe.moe_workspace_size(p, c) for c in range(6)}
    assert all(v >= 256 for v in sizes.values())
    assert sizes[moe.MOE_CALL_FORWARD] > sizes[moe.MOE_CALL_ROUTE]
    big = problem(T=4096)
    assert moe.moe_workspace_size(big, moe.MOE_CALL_FORWARD) > sizes[moe.MOE_CALL_FORWARD]
    # unsupported shapes report 0
    for bad in (problem(H=100), problem(I=96), problem(E=300), problem(top_k=17),
                problem(E=64, top_k=33), problem(num_shared=2), problem(T=-1)):
        assert moe.moe_workspace_size(bad, moe.MOE_CALL_FORWARD) == 0
    assert moe.moe_workspace_size(p, 42) == 0


def test_forward_workspace_covers_the_prefill_buffers(lib):
    c = CONFIGS["hy4_prefill"]
    p = moe.MoEProblem.from_config(c)
    n = moe.moe_workspace_size(p, moe.MOE_CALL_FORWARD)
    T, H, E, I, k = c.T, c.H, c.E, c.I, c.top_k
    # x_perm + h_perm + the weighted expert rows (which share their region with
    # the fp32 token accumulator of the scatter-add combine)
    must = T * k * H * 2 + T * (k + 1) * I * 2 + max(T * (k + 1) * H * 2, T * H * 4)
    assert must <= n < must * 1.1


def _call_forward(lib, pc, ws_ptr, ws_bytes, x=1 << 20):
    P = ctypes.c_void_p
    return lib.moe_forward(ctypes.byref(pc), P(x), P(x), None, P(x), P(x), P(x), None, None,
                           P(ws_ptr), ws_bytes, None)


def test_host_validation_rejects_before_launch(lib):
    # fake, never-dereferenced 16-byte-aligned addresses: every call below must
    # be rejected on the host, before anything reaches the GPU
    pc = problem().c()
    ws_need = moe.moe_workspace_size(problem(), moe.MOE_CALL_FORWARD)
    assert _call_forward(lib, pc, 1 << 24, ws_need - 1) == moe.MOE_ERR_WORKSPACE
    assert _call_forward(lib, pc, 0, ws_need) == moe.MOE_ERR_INVALID_ARG
    assert _call_forward(lib, pc, (1 << 24) + 8, ws_need) == moe.MOE_ERR_INVALID_ARG
    bad = problem(H=100).c()
    assert _call_forward(lib, bad, 1 << 24, ws_need) == moe.MOE_ERR_UNSUPPORTED
    nan_scale = problem(routed_scale=float("nan")).c()
    assert _call_forward(lib, nan_scale, 1 << 24, ws_need) == moe.MOE_ERR_INVALID_ARG
    # shared expert requested but no weights given
    P = ctypes.c_void_p
    x = 1 << 20
    rc = lib.moe_forward(ctypes.byref(pc), P(x), P(x), None, P(x), None, P(x), None, None,
                         P(1 << 24), ws_need, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    # an empty batch is a valid no-op that launches nothing
    before = moe.moe_launch_count()
    empty = problem(T=0).c()
    assert _call_forward(lib, empty, 1 << 24, moe.moe_workspace_size(problem(T=0), 5)) == 0
    assert moe.moe_launch_count() == before


def test_ffn_and_permute_validation(lib):
    pc = problem().c()
    P = ctypes.c_void_p
    ws = moe.moe_workspace_size(problem(), moe.MOE_CALL_FFN)
    x = 1 << 20
    assert lib.moe_grouped_swiglu_ffn(ctypes.byref(pc), P(x), 64, P(x), 0, P(x), P(x),
                                      P(1 << 24), ws, None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_grouped_swiglu_ffn(ctypes.byref(pc), P(x), 64, P(x), 257, P(x), P(x),
                                      P(1 << 24), ws, None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_grouped_swiglu_ffn(ctypes.byref(pc), None, 64, P(x), 4, P(x), P(x),
                                      P(1 << 24), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.byref(pc), None, P(x), P(x), P(x), P(x), P(x), P(1 << 24),
                           1 << 20, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(ctypes.byref(pc), P(x), P(x), None, P(x), P(x), P(1 << 24), 0,
                         None) == moe.MOE_ERR_WORKSPACE


def test_fp8_weight_encoder_validation(lib):
    # fake, never-dereferenced addresses: refused on the host before any launch
    # (the row encoder reads 16-byte vectors of w and writes 8-byte groups of q)
    p = problem(H=256, I=256).c()
    P = ctypes.c_void_p
    a = 1 << 20
    before = moe.moe_launch_count()

    def enc(pc, n, w, q):
        return lib.moe_quantize_weights_fp8(ctypes.byref(pc), n, P(w), P(q), P(a), P(a), None)

    assert enc(p, 2, a + 2, a) == moe.MOE_ERR_INVALID_ARG      # w not 16-byte aligned
    assert enc(p, 2, a, a + 8) == moe.MOE_ERR_INVALID_ARG      # q not 16-byte aligned
    assert enc(p, 0, a, a) == moe.MOE_ERR_INVALID_ARG          # no experts
    assert enc(problem(H=192, I=256).c(), 2, a, a) == moe.MOE_ERR_UNSUPPORTED
    assert moe.moe_launch_count() == before


def test_binding_refuses_cpu_tensors(lib):
    p = problem(T=4, H=64, I=64, E=2, top_k=1, num_shared=0)
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.moe_router_logits(p, x, x, torch.zeros(4, 2), torch.zeros(256, dtype=torch.uint8))


def test_missing_library_fails_loudly(tmp_path):
    """Without the CUDA library there is nothing to fall back to: loading it
    from a path where it does not exist raises, naming the build step."""
    import importlib
    fresh = importlib.reload(moe)  # a module instance with no library loaded yet
    try:
        with pytest.raises(RuntimeError, match="no non-CUDA implementation"):
            fresh.load_library(str(tmp_path / "libmoe_b200.so"))
    finally:
        importlib.reload(moe)


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """A C99 program using include/moe.h links against the library and runs
    its host-only calls (no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c_api", "c_api_check.c")
    exe = str(tmp_path / "c_api_check")
    libdir = os.path.dirname(moe.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        src, "-o", exe, "-L", libdir, "-lmoe_b200", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_binding_refuses_tensors_smaller_than_the_problem(lib):
    # The kernels take every extent from the problem, so the binding must
    # refuse an operand with fewer elements than the problem implies before
    # the C call (on CPU tensors the size check comes before the device check).
    p = problem(T=64, H=256, E=16, I=128, top_k=2, num_shared=1)
    T, H, E, I, k = p.T, p.H, p.E, p.I, p.top_k
    bf = torch.bfloat16
    full = dict(x=torch.zeros(T, H, dtype=bf), gate_w=torch.zeros(E, H, dtype=bf),
                expert_w=torch.zeros(E, 3, I, H, dtype=bf),
                shared_w=torch.zeros(3, I, H, dtype=bf), out=torch.zeros(T, H, dtype=bf),
                idx=torch.zeros(T, k, dtype=torch.int32), w=torch.zeros(T, k))
    before = moe.moe_launch_count()
    for name in full:
        args = dict(full)
        args[name] = args[name].reshape(-1)[:-1]  # one element short
        with pytest.raises(ValueError, match="elements"):
            moe.moe_forward(p, args["x"], args["gate_w"], None, args["expert_w"],
                            args["shared_w"], args["out"], args["idx"], args["w"],
                            torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="elements"):
        moe.moe_route(p, full["x"], full["gate_w"], torch.zeros(E - 1), full["idx"], full["w"],
                      torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="elements"):
        moe.moe_permute(p, full["idx"], full["x"], torch.zeros(E, dtype=torch.int32),
                        torch.zeros(T * k, dtype=torch.int32),
                        torch.zeros(T * k, dtype=torch.int32),
                        torch.zeros(T * k, H, dtype=bf), torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="elements"):
        moe.moe_combine(p, torch.zeros(T * k - 1, H, dtype=bf),
                        torch.zeros(T * k, dtype=torch.int32), full["w"], None, full["out"],
                        torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="elements"):
        moe.moe_grouped_swiglu_ffn(p, torch.zeros(10, H, dtype=bf),
                                   torch.zeros(E + 1, dtype=torch.int32), E,
                                   full["expert_w"], torch.zeros(9, H, dtype=bf),
                                   torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="elements"):
        moe.moe_forward_fp8(p, full["x"], full["gate_w"], None,
                            torch.zeros(E * 3 * I * H, dtype=torch.uint8),
                            torch.zeros(E * 2 * I), torch.zeros(E * H - 1),
                            None, None, None, full["out"], None, None,
                            torch.zeros(256, dtype=torch.uint8))
    assert moe.moe_launch_count() == before


def test_expert_tile_rows_query(lib):
    # host-only query of the token-tile widths of the expert GEMMs
    expect = {"tiny": 16, "hy3": 160, "hy4_prefill": 160, "hy4_decode": 16, "hy4_skew": 256}
    for name, width in expect.items():
        gu, dn = moe.moe_expert_tile_rows(moe.MoEProblem.from_config(CONFIGS[name]))
        assert (gu, dn) == (width, width), name
    with pytest.raises(moe.MoEError):
        moe.moe_expert_tile_rows(problem(H=100))


def test_schedule_cover_tokens_covers_every_chunk():
    import sys
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numpy as np
    from parity_util import chunk_bounds, schedule_cover_tokens
    for rows in (1, 15, 16, 17, 100, 160, 161, 320, 321, 16232):
        for width in (16, 32, 160, 256):
            b = chunk_bounds(rows, width)
            # contiguous, complete, at most `width` rows, multiples of 16 but the last
            assert b[0][0] == 0 and b[-1][1] == rows - 1
            for (f0, l0), (f1, _) in zip(b, b[1:]):
                assert f1 == l0 + 1 and (l0 - f0 + 1) % 16 == 0
            assert all(l - f + 1 <= width for f, l in b)
            assert len(b) == -(-rows // width)
    g = np.random.default_rng(0)
    T, E, k = 700, 12, 3
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)])
    toks, tiles = schedule_cover_tokens(idx, E, 1, (32, 160))
    for width in (32, 160):
        n = 0
        for e in range(E + 1):
            rows = [t for t in range(T) if e == E or e in idx[t]]
            for f, l in chunk_bounds(len(rows), width):
                assert rows[f] in toks and rows[l] in toks
                n += 1
        assert tiles[width] == n
