"""CPU tests of the C-ABI library: it loads, exports every entry point that
include/muonclip.h declares, rejects bad arguments before touching memory or the
GPU, and its host-side tile scheduler covers every output element."""
import ctypes
import os
import re
import subprocess

import pytest

import matrix_orthogonalising_optimizer_step_b200 as mc
from matrix_orthogonalising_optimizer_step_b200 import build as mcbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muonclip.h")


@pytest.fixture(scope="module")
def lib():
    mcbuild.build()
    return mc.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mc_\w+)\s*\(", text)))


def test_header_declares_the_three_operations():
    names = declared_functions()
    for n in ("mc_muon_step", "mc_qk_max_logit", "mc_qk_clip"):
        assert n in names


def test_binding_structures_match_the_header(lib):
    """The ctypes layouts of the binding have the sizes of the C structures
    the library was built with (a field added on one side only fails here)."""
    for which, cls in enumerate((mc.McParam, mc.McHparams, mc.McNormuon, mc.McClipSlice, mc.McKernelStat)):
        assert lib.mc_struct_size(which) == ctypes.sizeof(cls), cls.__name__
    assert lib.mc_struct_size(5) == 0


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(mc.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", mc.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (mc_\w+)$", out, flags=re.M))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
    # internal symbols stay hidden
    assert not any(s.startswith("_ZN2mc") for s in re.findall(r"\bT (\S+)$", out, flags=re.M))


def _params(n, rows=64, cols=96, base=0x100000):
    arr = (mc.McParam * max(n, 1))()
    for i in range(n):
        off = base + i * 0x10000
        arr[i] = mc.McParam(off, off + 0x4000, off + 0x8000, rows, cols, mc.MC_BF16, mc.MC_BF16, None)
    return arr


def test_argument_errors_return_codes_without_a_gpu(lib):
    hp = mc.make_hparams()
    P = ctypes.byref
    arr = _params(2)
    # null params with n > 0
    assert lib.mc_muon_step(None, 2, P(hp), None, 0, None, None) == mc.MC_ERR_INVAL
    assert "params" in mc.last_error()
    # negative n, null hp, bad ns_steps, bad eps
    assert lib.mc_muon_step(arr, -1, P(hp), None, 0, None, None) == mc.MC_ERR_INVAL
    assert lib.mc_muon_step(arr, 2, None, None, 0, None, None) == mc.MC_ERR_INVAL
    for bad in (dict(ns_steps=0), dict(ns_steps=100), dict(eps=0.0), dict(lr=float("nan"))):
        h = mc.make_hparams(**bad)
        assert lib.mc_muon_step(arr, 2, P(h), None, 0, None, None) == mc.MC_ERR_INVAL
    # bad shape, bad dtype, aliasing, misalignment
    a = _params(1); a[0].rows = 0
    assert lib.mc_muon_step(a, 1, P(hp), None, 0, None, None) == mc.MC_ERR_INVAL
    a = _params(1); a[0].w_dtype = 7
    assert lib.mc_muon_step(a, 1, P(hp), None, 0, None, None) == mc.MC_ERR_INVAL
    a = _params(1); a[0].m = a[0].w
    assert lib.mc_muon_step(a, 1, P(hp), None, 0, None, None) == mc.MC_ERR_INVAL
    a = _params(1); a[0].g = a[0].g + 2
    assert lib.mc_muon_step(a, 1, P(hp), None, 0, None, None) == mc.MC_ERR_ALIGN
    # a device (lr, wd) pair must be 4-byte aligned (its values are the caller's)
    h = mc.make_hparams(); h.lr_wd = 0x900002
    assert lib.mc_muon_step(arr, 2, P(h), None, 0, None, None) == mc.MC_ERR_ALIGN
    assert lib.mc_muon_workspace_size(arr, 2, P(h)) == 0
    # n == 0 is a no-op
    assert lib.mc_muon_step(arr, 0, P(hp), None, 0, None, None) == mc.MC_OK
    # QK
    assert lib.mc_qk_max_logit(None, None, None, 1, 8, 64, 2, 64, 1, None, None, 0, None) == mc.MC_ERR_INVAL
    assert lib.mc_qk_max_logit(16, 32, 48, 1, 8, 60, 2, 64, 1, 64, None, 0, None) == mc.MC_ERR_INVAL  # D % 8
    assert lib.mc_qk_max_logit(16, 32, 48, 1, 8, 64, 2, 64, 1, 66, None, 0, None) == mc.MC_ERR_ALIGN
    assert lib.mc_qk_clip(16, 32, 2, 8, 64, 48, 100.0, 1.5, None, None, None) == mc.MC_ERR_INVAL  # alpha
    assert lib.mc_qk_clip(16, 32, 2, 8, 64, 48, -1.0, 0.5, None, None, None) == mc.MC_ERR_INVAL   # tau
    assert lib.mc_qk_clip(16, 16, 2, 8, 64, 48, 100.0, 0.5, None, None, None) == mc.MC_ERR_INVAL  # alias
    assert lib.mc_qk_clip(16, 32, 2, 8, 64, 50, 100.0, 0.5, None, None, None) == mc.MC_ERR_ALIGN


def test_workspace_queries(lib):
    hp = mc.make_hparams()
    P = ctypes.byref
    one = lib.mc_muon_workspace_size(_params(1), 1, P(hp))
    two = lib.mc_muon_workspace_size(_params(2), 2, P(hp))
    assert one > 0 and two > one
    # 64 x 96 bf16: two bf16 iterates + the lo half + A, B (64 x 64 bf16)
    assert one >= 64 * 96 * (2 + 2 + 2) + 2 * 64 * 64 * 2
    tall = _params(1, rows=96, cols=64)
    assert lib.mc_muon_workspace_size(tall, 1, P(hp)) == one  # same bytes, stored layout
    assert lib.mc_muon_workspace_size(_params(1), 1, P(mc.make_hparams(ns_steps=0))) == 0
    q = lib.mc_qk_workspace_size(4, 4096, 4096, 32, 128)
    assert q >= 2 * 4 * 4096 * 4096 * 2
    assert lib.mc_qk_workspace_size(1, 8, 63, 1, 8) == 0


def test_tile_scheduler_host_check(tmp_path):
    src = os.path.join(ROOT, "tests", "host", "sched_check.cu")
    exe = tmp_path / "sched_check"
    cmd = [mcbuild.nvcc_path(), "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", mcbuild.CSRC, "-o", str(exe), src]
    subprocess.run(cmd, check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "OK", out.stdout


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mc, "_lib", None)
    monkeypatch.setattr(mc, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mc.load_library()


def test_coefficient_table_validation(lib):
    P = ctypes.byref
    bad = mc.make_hparams(ns_steps=2, coeffs=[(1.5, float("nan"), 0.0), (2.0, -1.5, 0.5)])
    assert lib.mc_muon_step(_params(1), 1, P(bad), None, 0, None, None) == mc.MC_ERR_INVAL
    assert "coeffs" in mc.last_error()
    with pytest.raises(ValueError):
        mc.make_hparams(ns_steps=3, coeffs=[(1.5, -0.5, 0.0)])


def _slice(w=0x100000, r0=0, r1=8, cols=64, dtype=mc.MC_BF16, head=0, e=0.5, reserved=0):
    return mc.McClipSlice(w, r0, r1, cols, dtype, head, e, reserved)


def test_clip_slices_argument_errors(lib):
    def call(slices, n=None, smax=0x200000, H=4, tau=100.0):
        arr = (mc.McClipSlice * max(len(slices), 1))(*slices)
        return lib.mc_qk_clip_slices(arr, len(slices) if n is None else n, smax, H, tau, None, None, None)

    ok = _slice()
    assert lib.mc_qk_clip_slices(None, 1, 0x200000, 4, 100.0, None, None, None) == mc.MC_ERR_INVAL
    assert call([ok], n=-1) == mc.MC_ERR_INVAL
    assert call([ok], smax=0) == mc.MC_ERR_INVAL
    assert call([ok], H=0) == mc.MC_ERR_INVAL
    assert call([ok], tau=0.0) == mc.MC_ERR_INVAL
    assert call([ok], tau=float("inf")) == mc.MC_ERR_INVAL
    assert call([_slice(w=0)]) == mc.MC_ERR_INVAL
    assert call([_slice(dtype=5)]) == mc.MC_ERR_INVAL
    assert call([_slice(r0=8, r1=8)]) == mc.MC_ERR_INVAL
    assert call([_slice(r0=-1)]) == mc.MC_ERR_INVAL
    assert call([_slice(cols=0)]) == mc.MC_ERR_INVAL
    assert call([_slice(head=4)]) == mc.MC_ERR_INVAL
    assert call([_slice(head=-1)]) == mc.MC_ERR_INVAL
    assert call([_slice(e=1.5)]) == mc.MC_ERR_INVAL
    assert call([_slice(e=float("nan"))]) == mc.MC_ERR_INVAL
    assert call([_slice(reserved=1)]) == mc.MC_ERR_INVAL
    assert call([_slice(w=0x100008)]) == mc.MC_ERR_ALIGN
    assert lib.mc_qk_clip_slices((mc.McClipSlice * 1)(ok), 1, 0x200004, 4, 100.0, None, None, None) == mc.MC_ERR_ALIGN
    # overlapping rows of one matrix, and two base pointers whose ranges meet
    assert call([_slice(r0=0, r1=8), _slice(r0=7, r1=9, head=1)]) == mc.MC_ERR_INVAL
    assert "overlap" in mc.last_error()
    assert call([_slice(r0=0, r1=8), _slice(w=0x100000 + 7 * 128, r0=0, r1=1, head=1)]) == mc.MC_ERR_INVAL
    # smax is required even for an empty map
    assert call([], n=0, smax=0) == mc.MC_ERR_INVAL


def test_mla_argument_errors_and_workspace(lib):
    a = (0x100000, 0x200000, 0x300000, 0x400000, 0x500000)
    args = lambda **k: dict(dict(B=1, S=64, D=64, H=2, dc=64, dr=32, causal=1), **k)

    def call(ptrs=a, smax=0x600000, **k):
        d = args(**k)
        return lib.mc_mla_max_logit(*ptrs, d["B"], d["S"], d["D"], d["H"], d["dc"], d["dr"], d["causal"],
                                    smax, None, 0, None)
    assert call(dc=32) == mc.MC_ERR_INVAL          # dc must be a multiple of 64
    assert call(dr=12) == mc.MC_ERR_INVAL          # dr multiple of 8
    assert call(dr=0) == mc.MC_ERR_INVAL
    assert call(D=60) == mc.MC_ERR_INVAL
    assert call(ptrs=(0,) + a[1:]) == mc.MC_ERR_INVAL
    assert call(smax=0) == mc.MC_ERR_INVAL
    assert call(ptrs=a[:4] + (0x500008,)) == mc.MC_ERR_ALIGN
    n = lib.mc_mla_workspace_size(2, 128, 64, 4, 128, 64)
    bs = 2 * 128
    assert n >= 2 * bs * (2 * 4 * 128 + 4 * 64 + 64) + 4 * 4
    assert lib.mc_mla_workspace_size(2, 128, 64, 4, 96, 64) == 0


def test_normuon_argument_errors(lib):
    P = ctypes.byref
    hp = mc.make_hparams()
    arr = _params(2)
    vptrs = (ctypes.c_void_p * 2)(0x900000, 0x910000)
    good = mc.McNormuon(0.95, 1e-8, ctypes.cast(vptrs, ctypes.c_void_p).value)
    call = lambda nm: lib.mc_normuon_step(arr, 2, P(hp), nm, None, 0, None, None)
    assert call(None) == mc.MC_ERR_INVAL
    for b2, eps in ((1.0, 1e-8), (-0.1, 1e-8), (float("nan"), 1e-8), (0.9, -1.0), (0.9, float("inf"))):
        assert call(P(mc.McNormuon(b2, eps, good.v))) == mc.MC_ERR_INVAL
    assert call(P(mc.McNormuon(0.95, 1e-8, None))) == mc.MC_ERR_INVAL
    bad = (ctypes.c_void_p * 2)(0x900000, 0)
    assert call(P(mc.McNormuon(0.95, 1e-8, ctypes.cast(bad, ctypes.c_void_p).value))) == mc.MC_ERR_INVAL
    alias = (ctypes.c_void_p * 2)(arr[0].m, 0x910000)
    assert call(P(mc.McNormuon(0.95, 1e-8, ctypes.cast(alias, ctypes.c_void_p).value))) == mc.MC_ERR_INVAL
    mis = (ctypes.c_void_p * 2)(0x900004, 0x910000)
    assert call(P(mc.McNormuon(0.95, 1e-8, ctypes.cast(mis, ctypes.c_void_p).value))) == mc.MC_ERR_ALIGN
    # the workspace adds two fp32 row arrays and the row table to the Muon plan
    a = lib.mc_muon_workspace_size(arr, 2, P(hp))
    b = lib.mc_normuon_workspace_size(arr, 2, P(hp))
    assert b >= a + 2 * 4 * (64 + 64)


def test_polar_express_coeffs_match_the_oracle(lib):
    import numpy as np
    import oracle
    for steps, l0, safety in ((10, 1e-3, 0.01), (5, 1e-3, 0.01), (8, 1e-2, 0.0), (3, 0.3, 0.02)):
        got = np.array(mc.polar_express_coeffs(steps, l0, safety))
        want = np.array(oracle.polar_express_schedule(steps, l0, safety))
        assert got.shape == (steps, 3)
        assert np.allclose(got, want, rtol=1e-6, atol=1e-6), (steps, l0, safety)
    # the printed effect, through the library's own table
    assert float(oracle.phi_schedule(1e-4, mc.polar_express_coeffs(10))) == pytest.approx(0.994, abs=5e-4)
    out = (ctypes.c_float * 3)()
    assert lib.mc_polar_express_coeffs(0, 1e-3, 0.01, out) == mc.MC_ERR_INVAL
    assert lib.mc_polar_express_coeffs(5, 1.0, 0.01, out) == mc.MC_ERR_INVAL
    assert lib.mc_polar_express_coeffs(5, 1e-3, -0.1, out) == mc.MC_ERR_INVAL
    assert lib.mc_polar_express_coeffs(5, 1e-3, 0.01, None) == mc.MC_ERR_INVAL


def test_host_grads_entry_arguments_and_workspace(lib):
    P = ctypes.byref
    hp = mc.make_hparams()
    arr = _params(6, rows=128, cols=256)
    hptr = (ctypes.c_void_p * 6)(*[0x7000000 + i * 0x100000 for i in range(6)])
    assert lib.mc_muon_step_host_grads(arr, hptr, 6, P(hp), 0, None, 0, None, None) == mc.MC_ERR_INVAL
    assert lib.mc_muon_step_host_grads(arr, None, 6, P(hp), 2, None, 0, None, None) == mc.MC_ERR_INVAL
    bad = (ctypes.c_void_p * 6)(*([0x7000000] * 5 + [0]))
    assert lib.mc_muon_step_host_grads(arr, bad, 6, P(hp), 2, None, 0, None, None) == mc.MC_ERR_INVAL
    # one compute region reused by every piece, plus every piece's own tables:
    # with a single piece both entry points plan the same workspace
    full = lib.mc_muon_workspace_size(arr, 6, P(hp))
    one = lib.mc_muon_host_grads_workspace_size(arr, 6, P(hp), 1)
    assert full == one
    # six equal matrices: the ramp starts below one matrix, so every piece holds one
    three = lib.mc_muon_host_grads_workspace_size(arr, 6, P(hp), 3)
    single = lib.mc_muon_workspace_size(arr, 1, P(hp))
    assert single < three <= single + 64 * 1024 and three < one
    assert lib.mc_muon_host_grads_workspace_size(arr, 6, P(hp), 0) == 0


def test_product_never_imports_the_oracle():
    """The library package (binding, sharded step, workloads, build) has no
    path to oracle/: the oracle is test infrastructure only."""
    pkg = os.path.join(ROOT, "matrix_orthogonalising_optimizer_step_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "oracle." not in re.sub(r"#.*|\"\"\".*?\"\"\"", "", text, flags=re.S), f


def test_binding_rejects_cpu_tensors_without_computing():
    """No CPU fallback: host tensors are refused before anything runs."""
    import torch
    W = torch.zeros(8, 16, dtype=torch.bfloat16)
    G = torch.zeros(8, 16, dtype=torch.bfloat16)
    M = torch.zeros(8, 16)
    with pytest.raises(ValueError, match="CUDA"):
        mc.muon_step([W], [G], [M])
    X = torch.zeros(1, 4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        mc.qk_max_logit(X, torch.zeros(16, 16, dtype=torch.bfloat16), torch.zeros(16, 16, dtype=torch.bfloat16), 2, 8)


def test_bounded_wait_selftest_rejects_bad_limits(lib):
    """The limit is checked on the host before anything is launched."""
    for bad in (0, 999, -5, (1 << 32) + 1):
        assert lib.mc_selftest_bounded_wait(bad, None) == mc.MC_ERR_INVAL
        assert "limit_cycles" in mc.last_error()
