"""B200-native MuonClip step: Python binding over the C ABI in include/muonclip.h.

The binding only marshals arguments: every step of the Muon update and of
QK-Clip runs in the sm_100a kernels of ``libmuonclip.so``.  PyTorch supplies
device memory and the current stream.  There is no fallback: if the library is
missing or the device is not a B200 the calls raise.

    from matrix_orthogonalising_optimizer_step_b200 import muon_step, qk_max_logit, qk_clip

Also: muon_step_host_grads, normuon_step, mla_max_logit, qk_clip_slices (with
mla_slices), polar_express_coeffs, shard_plan, qk_max_logit_static, and the
data-parallel step in ``sharded``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmuonclip.so")

MC_OK, MC_ERR_INVAL, MC_ERR_ALIGN, MC_ERR_NOSPC, MC_ERR_CUDA, MC_ERR_UNSUPPORTED, MC_ERR_DEVICE, MC_ERR_NONFINITE = (
    0, -1, -2, -3, -4, -5, -6, -7)
MC_F32, MC_BF16 = 0, 1

# Names the C ABI exports (include/muonclip.h).
EXPORTS = ("mc_muon_workspace_size", "mc_muon_step", "mc_qk_workspace_size", "mc_qk_max_logit",
           "mc_qk_clip", "mc_last_error", "mc_device_status", "mc_profile_begin", "mc_profile_end",
           "mc_qk_max_logit_static", "mc_qk_clip_slices", "mc_mla_workspace_size", "mc_mla_max_logit",
           "mc_shard_plan", "mc_normuon_workspace_size", "mc_normuon_step", "mc_polar_express_coeffs",
           "mc_muon_host_grads_workspace_size", "mc_muon_step_host_grads", "mc_selftest_bounded_wait",
           "mc_struct_size")
MC_QK_STATIC_MAX_ELEMS = 1 << 24
MC_QK_STATIC_MAX_HEADS = 4096


class McParam(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("g", ctypes.c_void_p), ("m", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("w_dtype", ctypes.c_int32), ("g_dtype", ctypes.c_int32),
                ("update_out", ctypes.c_void_p)]


class McHparams(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_float), ("nesterov", ctypes.c_int32), ("lr", ctypes.c_float),
                ("wd", ctypes.c_float), ("ns_steps", ctypes.c_int32), ("a", ctypes.c_float),
                ("b", ctypes.c_float), ("c", ctypes.c_float), ("eps", ctypes.c_float),
                ("rms_scale", ctypes.c_float), ("coeffs", ctypes.c_void_p), ("lr_wd", ctypes.c_void_p)]


class McNormuon(ctypes.Structure):
    _fields_ = [("beta2", ctypes.c_float), ("eps", ctypes.c_float), ("v", ctypes.c_void_p)]


class McClipSlice(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("row_begin", ctypes.c_int64), ("row_end", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("dtype", ctypes.c_int32), ("head", ctypes.c_int32),
                ("exponent", ctypes.c_float), ("reserved", ctypes.c_int32)]


class McKernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("flops_executed", ctypes.c_double),
                ("flops_dense_equiv", ctypes.c_double), ("bytes", ctypes.c_double)]


class MuonClipError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


_lib = None


def load_library():
    """Load libmuonclip.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m matrix_orthogonalising_optimizer_step_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.mc_muon_workspace_size.argtypes = [P(McParam), i32, P(McHparams)]
    lib.mc_muon_workspace_size.restype = sz
    lib.mc_muon_step.argtypes = [P(McParam), i32, P(McHparams), vp, sz, vp, vp]
    lib.mc_muon_step.restype = i32
    lib.mc_qk_workspace_size.argtypes = [i32] * 5
    lib.mc_qk_workspace_size.restype = sz
    lib.mc_qk_max_logit.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, sz, vp]
    lib.mc_qk_max_logit.restype = i32
    lib.mc_qk_clip.argtypes = [vp, vp, i32, i32, i32, vp, ctypes.c_float, ctypes.c_float, vp, vp, vp]
    lib.mc_qk_clip.restype = i32
    lib.mc_last_error.argtypes = []
    lib.mc_last_error.restype = ctypes.c_char_p
    lib.mc_device_status.argtypes = []
    lib.mc_device_status.restype = i32
    lib.mc_qk_max_logit_static.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
    lib.mc_qk_max_logit_static.restype = i32
    lib.mc_qk_clip_slices.argtypes = [P(McClipSlice), i32, vp, i32, ctypes.c_float, vp, vp, vp]
    lib.mc_qk_clip_slices.restype = i32
    lib.mc_mla_workspace_size.argtypes = [i32] * 6
    lib.mc_mla_workspace_size.restype = sz
    lib.mc_mla_max_logit.argtypes = [vp, vp, vp, vp, vp] + [i32] * 7 + [vp, vp, sz, vp]
    lib.mc_mla_max_logit.restype = i32
    lib.mc_normuon_workspace_size.argtypes = [P(McParam), i32, P(McHparams)]
    lib.mc_normuon_workspace_size.restype = sz
    lib.mc_normuon_step.argtypes = [P(McParam), i32, P(McHparams), P(McNormuon), vp, sz, vp, vp]
    lib.mc_normuon_step.restype = i32
    lib.mc_muon_host_grads_workspace_size.argtypes = [P(McParam), i32, P(McHparams), i32]
    lib.mc_muon_host_grads_workspace_size.restype = sz
    lib.mc_muon_step_host_grads.argtypes = [P(McParam), vp, i32, P(McHparams), i32, vp, sz, vp, vp]
    lib.mc_muon_step_host_grads.restype = i32
    lib.mc_polar_express_coeffs.argtypes = [i32, ctypes.c_double, ctypes.c_double, P(ctypes.c_float)]
    lib.mc_polar_express_coeffs.restype = i32
    lib.mc_shard_plan.argtypes = [P(ctypes.c_int64), P(ctypes.c_int64), i32, i32, i32, P(ctypes.c_int32),
                                  P(ctypes.c_double)]
    lib.mc_shard_plan.restype = i32
    lib.mc_selftest_bounded_wait.argtypes = [ctypes.c_longlong, vp]
    lib.mc_selftest_bounded_wait.restype = i32
    lib.mc_struct_size.argtypes = [i32]
    lib.mc_struct_size.restype = sz
    lib.mc_profile_begin.argtypes = []
    lib.mc_profile_begin.restype = i32
    lib.mc_profile_end.argtypes = [P(McKernelStat), i32, P(ctypes.c_int)]
    lib.mc_profile_end.restype = i32
    _lib = lib
    return lib


def _check(rc: int):
    if rc != MC_OK:
        raise MuonClipError(rc, load_library().mc_last_error().decode())


def last_error() -> str:
    return load_library().mc_last_error().decode()


def device_status() -> int:
    """Synchronise the current device and return (and clear) the library's
    device error word: MC_OK, MC_ERR_DEVICE (a bounded wait ran out) or
    MC_ERR_NONFINITE (a Muon step met a NaN/Inf gradient or momentum)."""
    return load_library().mc_device_status()


def profile_begin() -> None:
    """Start bracketing every kernel this thread's calls launch with CUDA events."""
    _check(load_library().mc_profile_begin())


def profile_end() -> dict:
    """Stop profiling; returns {kernel kind: {launches, total_ms, flops,
    flops_executed, flops_dense_equiv, bytes}} of device time and work."""
    lib = load_library()
    rows = (McKernelStat * 32)()
    n = ctypes.c_int(0)
    _check(lib.mc_profile_end(rows, 32, ctypes.byref(n)))
    out = {}
    for i in range(min(n.value, 32)):
        r = rows[i]
        out[r.name.decode()] = dict(launches=int(r.launches), total_ms=float(r.total_ms), flops=float(r.flops),
                                    flops_executed=float(r.flops_executed),
                                    flops_dense_equiv=float(r.flops_dense_equiv), bytes=float(r.bytes))
    return out


# ----------------------------------------------------------------- helpers
def _torch():
    import torch
    return torch


def _stream_handle(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return MC_F32
    if t.dtype == torch.bfloat16:
        return MC_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _need_cuda_contig(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _one_device(tensors):
    """The device every (non-None) tensor lives on; raises if they differ.
    Each C call runs with that device current, so the library's per-device
    state, the stream and the pointers all belong to it."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all tensors must be on one CUDA device, got {sorted(str(d) for d in devs)}")
    return devs.pop()


def _check_qk_args(x, wq, wk, H, dh, smax_out, names=("x", "wq", "wk")):
    """Shapes of the MHA S_max call: x [B, S, D] and wq, wk [H*dh, D], bf16,
    contiguous; smax_out (if given) fp32, contiguous, at least H entries."""
    torch = _torch()
    for t, nm in zip((x, wq, wk), names):
        _need_cuda_contig(t, nm)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{nm} must be bfloat16")
    if x.dim() != 3:
        raise ValueError(f"x must be 3-D [B, S, D], got shape {tuple(x.shape)}")
    want = (int(H) * int(dh), int(x.shape[2]))
    for t, nm in ((wq, names[1]), (wk, names[2])):
        if tuple(t.shape) != want:
            raise ValueError(f"{nm} must have shape (H*dh, D) = {want}, got {tuple(t.shape)}")
    _check_out(smax_out, "smax_out", torch.float32, H)


def _check_out(t, name, dtype, n):
    if t is None:
        return
    _need_cuda_contig(t, name)
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    if t.numel() < int(n):
        raise ValueError(f"{name} must hold at least {int(n)} entries, got {t.numel()}")


def make_hparams(mu=0.95, nesterov=True, lr=0.02, wd=0.1, ns_steps=5, a=3.4445, b=-4.7750,
                 c=2.0315, eps=1e-7, rms_scale=0.2, coeffs=None, lr_wd=None) -> McHparams:
    """``coeffs``: optional list of ns_steps (a_k, b_k, c_k) triples, one per
    Newton-Schulz iteration.  The returned struct keeps the coefficient array
    alive (as ``_coeff_buf``).  ``lr_wd``: optional CUDA float32 tensor of two
    elements (lr, wd) that the kernels read when they run, in place of ``lr``
    and ``wd`` (for a learning-rate schedule under a captured CUDA graph)."""
    h = McHparams(float(mu), int(bool(nesterov)), float(lr), float(wd), int(ns_steps),
                  float(a), float(b), float(c), float(eps), float(rms_scale), None, None)
    if lr_wd is not None:
        torch = _torch()
        if not (lr_wd.is_cuda and lr_wd.dtype == torch.float32 and lr_wd.is_contiguous() and lr_wd.numel() == 2):
            raise ValueError("lr_wd must be a contiguous CUDA float32 tensor of two elements (lr, wd)")
        h._lr_wd = lr_wd
        h.lr_wd = lr_wd.data_ptr()
    if coeffs is not None:
        flat = [float(v) for t in coeffs for v in t]
        if len(flat) != 3 * int(ns_steps):
            raise ValueError("coeffs must hold one (a, b, c) triple per Newton-Schulz step")
        buf = (ctypes.c_float * len(flat))(*flat)
        h._coeff_buf = buf
        h.coeffs = ctypes.cast(buf, ctypes.c_void_p)
    return h


def make_params(weights, grads, moms, update_outs=None):
    n = len(weights)
    if not (len(grads) == n and len(moms) == n):
        raise ValueError("weights, grads and moms must have the same length")
    arr = (McParam * max(n, 1))()
    for i in range(n):
        W, G, M = weights[i], grads[i], moms[i]
        for t, nm in ((W, "weight"), (G, "grad"), (M, "momentum")):
            _need_cuda_contig(t, f"{nm}[{i}]")
            if t.dim() != 2:
                raise ValueError(f"{nm}[{i}] must be 2D")
        if G.shape != W.shape or M.shape != W.shape:
            raise ValueError(f"shape mismatch at index {i}")
        if M.dtype != _torch().float32:
            raise TypeError(f"momentum[{i}] must be float32")
        U = update_outs[i] if update_outs is not None else None
        if U is not None:
            _need_cuda_contig(U, f"update_out[{i}]")
            if U.shape != W.shape or U.dtype != _torch().float32:
                raise ValueError(f"update_out[{i}] must be float32 of the weight's shape")
        arr[i] = McParam(_ptr(W), _ptr(G), _ptr(M), int(W.shape[0]), int(W.shape[1]),
                         _dtype_code(W), _dtype_code(G), _ptr(U))
    return arr, n


_workspaces = {}


def _workspace(tag, device, nbytes):
    """Device scratch owned by PyTorch's allocator, cached per (tag, device)."""
    torch = _torch()
    key = (tag, device)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        _workspaces.pop(key, None)
        ws = torch.empty(max(int(nbytes), 1024), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def release_workspaces():
    _workspaces.clear()


# ----------------------------------------------------------------- the API
def muon_workspace_size(weights, grads, moms, hparams: Optional[McHparams] = None, **hp) -> int:
    lib = load_library()
    arr, n = make_params(weights, grads, moms)
    h = hparams if hparams is not None else make_hparams(**hp)
    return int(lib.mc_muon_workspace_size(arr, n, ctypes.byref(h)))


def muon_step(weights: Sequence, grads: Sequence, moms: Sequence, *, norms_out=None,
              update_outs=None, workspace=None, stream=None, hparams: Optional[McHparams] = None,
              **hp) -> None:
    """One Muon step on every (W, G, M) triple, in place on W and M (see
    mc_muon_step in include/muonclip.h).  Keyword hyper-parameters: mu,
    nesterov, lr, wd, ns_steps, a, b, c, eps, rms_scale."""
    lib = load_library()
    arr, n = make_params(weights, grads, moms, update_outs)
    h = hparams if hparams is not None else make_hparams(**hp)
    if n == 0:
        return
    _check_out(norms_out, "norms_out", _torch().float32, n)
    dev = _one_device(list(weights) + list(grads) + list(moms) + list(update_outs or []) + [norms_out, workspace])
    need = int(lib.mc_muon_workspace_size(arr, n, ctypes.byref(h)))
    if need == 0:
        _check(lib.mc_muon_step(arr, n, ctypes.byref(h), None, 0, None, None))
    with _torch().cuda.device(dev):
        ws = workspace if workspace is not None else _workspace("muon", dev, need)
        _check(lib.mc_muon_step(arr, n, ctypes.byref(h), _ptr(ws), int(ws.numel() * ws.element_size()),
                                _ptr(norms_out), _stream_handle(stream)))


def muon_step_host_grads(weights: Sequence, grads: Sequence, grads_host: Sequence, moms: Sequence, *,
                         chunks: int = 8, norms_out=None, update_outs=None, workspace=None, stream=None,
                         hparams: Optional[McHparams] = None, **hp) -> None:
    """``muon_step`` whose gradients start in (page-locked) host memory:
    ``grads_host[i]`` is copied into the device tensor ``grads[i]`` piece by
    piece, overlapped with the step of the pieces already on the device (see
    mc_muon_step_host_grads).  Results are those of ``muon_step``."""
    lib = load_library()
    arr, n = make_params(weights, grads, moms, update_outs)
    if len(grads_host) != n:
        raise ValueError("one host gradient per matrix")
    hptr = (ctypes.c_void_p * max(n, 1))()
    for i, (gh, g) in enumerate(zip(grads_host, grads)):
        if gh.is_cuda or not gh.is_contiguous() or gh.dtype != g.dtype or gh.shape != g.shape:
            raise ValueError(f"grads_host[{i}] must be a contiguous CPU tensor shaped and typed like grads[{i}]")
        hptr[i] = _ptr(gh)
    h = hparams if hparams is not None else make_hparams(**hp)
    if n == 0:
        return
    _check_out(norms_out, "norms_out", _torch().float32, n)
    dev = _one_device(list(weights) + list(grads) + list(moms) + list(update_outs or []) + [norms_out, workspace])
    need = int(lib.mc_muon_host_grads_workspace_size(arr, n, ctypes.byref(h), int(chunks)))
    if need == 0:
        _check(lib.mc_muon_step_host_grads(arr, hptr, n, ctypes.byref(h), int(chunks), None, 0, None, None))
    with _torch().cuda.device(dev):
        ws = workspace if workspace is not None else _workspace("muon", dev, need)
        _check(lib.mc_muon_step_host_grads(arr, hptr, n, ctypes.byref(h), int(chunks), _ptr(ws),
                                           int(ws.numel() * ws.element_size()), _ptr(norms_out),
                                           _stream_handle(stream)))


def make_normuon(vs, beta2: float = 0.95, eps: float = 1e-8) -> McNormuon:
    """McNormuon over per-matrix row-state tensors ``vs`` (fp32 [rows], CUDA).
    The host pointer array is kept alive on the returned struct."""
    torch = _torch()
    ptrs = (ctypes.c_void_p * max(len(vs), 1))()
    for i, v in enumerate(vs):
        _need_cuda_contig(v, f"vs[{i}]")
        if v.dtype != torch.float32:
            raise TypeError(f"vs[{i}] must be float32")
        ptrs[i] = _ptr(v)
    nm = McNormuon(float(beta2), float(eps), ctypes.cast(ptrs, ctypes.c_void_p).value)
    nm._ptrs = ptrs
    return nm


def normuon_step(weights: Sequence, grads: Sequence, moms: Sequence, vs: Sequence, *, beta2: float = 0.95,
                 eps_v: float = 1e-8, norms_out=None, update_outs=None, workspace=None, stream=None,
                 hparams: Optional[McHparams] = None, **hp) -> None:
    """One NorMuon step (see mc_normuon_step in include/muonclip.h): the Muon
    step with each row of the orthogonalised update divided by the square root
    of its running second moment ``vs[i]`` (fp32 [rows], updated in place),
    then rescaled to the Frobenius norm it had."""
    lib = load_library()
    arr, n = make_params(weights, grads, moms, update_outs)
    if len(vs) != n:
        raise ValueError("one row-state tensor per matrix")
    for i, (v, w) in enumerate(zip(vs, weights)):
        if v.shape != (w.shape[0],):
            raise ValueError(f"vs[{i}] must have shape ({w.shape[0]},)")
    h = hparams if hparams is not None else make_hparams(**hp)
    nm = make_normuon(vs, beta2, eps_v)
    if n == 0:
        return
    _check_out(norms_out, "norms_out", _torch().float32, n)
    dev = _one_device(list(weights) + list(grads) + list(moms) + list(vs) + list(update_outs or []) +
                      [norms_out, workspace])
    need = int(lib.mc_normuon_workspace_size(arr, n, ctypes.byref(h)))
    if need == 0:
        _check(lib.mc_normuon_step(arr, n, ctypes.byref(h), ctypes.byref(nm), None, 0, None, None))
    with _torch().cuda.device(dev):
        ws = workspace if workspace is not None else _workspace("muon", dev, need)
        _check(lib.mc_normuon_step(arr, n, ctypes.byref(h), ctypes.byref(nm), _ptr(ws),
                                   int(ws.numel() * ws.element_size()), _ptr(norms_out), _stream_handle(stream)))


def qk_workspace_size(B, S, D, H, dh) -> int:
    return int(load_library().mc_qk_workspace_size(B, S, D, H, dh))


def qk_max_logit(x, wq, wk, H: int, dh: int, *, causal: bool = True, smax_out=None,
                 workspace=None, stream=None):
    """Per-head S_max (fp32 [H]) of causal attention with Q = x Wq^T, K = x Wk^T."""
    torch = _torch()
    lib = load_library()
    _check_qk_args(x, wq, wk, H, dh, smax_out)
    dev = _one_device([x, wq, wk, smax_out, workspace])
    B, S, D = x.shape
    if smax_out is None:
        smax_out = torch.empty(H, dtype=torch.float32, device=dev)
    need = int(lib.mc_qk_workspace_size(B, S, D, H, dh))
    if need == 0:
        _check(lib.mc_qk_max_logit(None, None, None, B, S, D, H, dh, int(causal), None, None, 0, None))
    with torch.cuda.device(dev):
        ws = workspace if workspace is not None else _workspace("qk", dev, need)
        _check(lib.mc_qk_max_logit(_ptr(x), _ptr(wq), _ptr(wk), B, S, D, H, dh, int(causal),
                                   _ptr(smax_out), _ptr(ws), int(ws.numel() * ws.element_size()),
                                   _stream_handle(stream)))
    return smax_out


def qk_clip(wq, wk, smax, H: int, dh: int, *, tau: float = 100.0, alpha: float = 0.5,
            gamma_out=None, mask_out=None, stream=None):
    """QK-Clip in place on Wq/Wk rows of heads with S_max > tau.  Returns
    (gamma [H] fp32, mask [H] int32)."""
    torch = _torch()
    lib = load_library()
    for t, nm in ((wq, "wq"), (wk, "wk")):
        _need_cuda_contig(t, nm)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{nm} must be bfloat16")
        if t.dim() != 2 or int(t.shape[0]) != int(H) * int(dh):
            raise ValueError(f"{nm} must have shape (H*dh, D) with H*dh = {int(H) * int(dh)}, got {tuple(t.shape)}")
    if wk.shape != wq.shape:
        raise ValueError("wq and wk must have the same shape")
    _check_out(smax, "smax", torch.float32, H)
    _check_out(gamma_out, "gamma_out", torch.float32, H)
    _check_out(mask_out, "mask_out", torch.int32, H)
    dev = _one_device([wq, wk, smax, gamma_out, mask_out])
    D = int(wq.shape[1])
    if gamma_out is None:
        gamma_out = torch.empty(H, dtype=torch.float32, device=dev)
    if mask_out is None:
        mask_out = torch.empty(H, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib.mc_qk_clip(_ptr(wq), _ptr(wk), H, dh, D, _ptr(smax), float(tau), float(alpha),
                              _ptr(gamma_out), _ptr(mask_out), _stream_handle(stream)))
    return gamma_out, mask_out


def make_clip_slices(slices):
    """ctypes array of McClipSlice from (weight, head, row_begin, row_end,
    exponent) tuples; each weight is a contiguous 2D CUDA tensor (bf16 or fp32)."""
    arr = (McClipSlice * max(len(slices), 1))()
    for i, (w, head, r0, r1, e) in enumerate(slices):
        _need_cuda_contig(w, f"slices[{i}] weight")
        if w.dim() != 2:
            raise ValueError(f"slices[{i}]: weight must be 2D")
        arr[i] = McClipSlice(_ptr(w), int(r0), int(r1), int(w.shape[1]), _dtype_code(w), int(head), float(e), 0)
    return arr, len(slices)


def mla_slices(wqc, wkc, wqr, H: int, dc: int, dr: int):
    """The MLA slice map: per head h, rows of the content query and key with
    exponent 1/2 and rows of the rotary query with exponent 1 (the shared
    rotary key has no entry, so it is never written)."""
    out = []
    for h in range(H):
        out += [(wqc, h, h * dc, (h + 1) * dc, 0.5), (wkc, h, h * dc, (h + 1) * dc, 0.5),
                (wqr, h, h * dr, (h + 1) * dr, 1.0)]
    return out


def qk_clip_slices(slices, smax, H: int, *, tau: float = 100.0, gamma_out=None, mask_out=None, stream=None):
    """QK-Clip in place over an explicit slice map (see mc_qk_clip_slices).
    Returns (gamma [H] fp32, mask [H] int32)."""
    torch = _torch()
    lib = load_library()
    _check_out(smax, "smax", torch.float32, H)
    _check_out(gamma_out, "gamma_out", torch.float32, H)
    _check_out(mask_out, "mask_out", torch.int32, H)
    arr, n = make_clip_slices(slices)
    dev = _one_device([smax, gamma_out, mask_out] + [sl[0] for sl in slices])
    if gamma_out is None:
        gamma_out = torch.empty(H, dtype=torch.float32, device=dev)
    if mask_out is None:
        mask_out = torch.empty(H, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib.mc_qk_clip_slices(arr, n, _ptr(smax), H, float(tau), _ptr(gamma_out), _ptr(mask_out),
                                     _stream_handle(stream)))
    return gamma_out, mask_out


def mla_workspace_size(B, S, D, H, dc, dr) -> int:
    return int(load_library().mc_mla_workspace_size(B, S, D, H, dc, dr))


def mla_max_logit(x, wqc, wkc, wqr, wkr, H: int, dc: int, dr: int, *, causal: bool = True, smax_out=None,
                  workspace=None, stream=None):
    """Per-head S_max (fp32 [H]) of multi-head latent attention: content part
    x W_qC^T . x W_kC^T per head plus rotary part x W_qR^T . x W_kR^T with one
    shared rotary key, over sqrt(dc + dr) (see mc_mla_max_logit)."""
    torch = _torch()
    lib = load_library()
    for t, nm in ((x, "x"), (wqc, "wqc"), (wkc, "wkc"), (wqr, "wqr"), (wkr, "wkr")):
        _need_cuda_contig(t, nm)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{nm} must be bfloat16")
    if x.dim() != 3:
        raise ValueError(f"x must be 3-D [B, S, D], got shape {tuple(x.shape)}")
    D = int(x.shape[2])
    for t, nm, rows in ((wqc, "wqc", H * dc), (wkc, "wkc", H * dc), (wqr, "wqr", H * dr), (wkr, "wkr", dr)):
        if tuple(t.shape) != (int(rows), D):
            raise ValueError(f"{nm} must have shape {(int(rows), D)}, got {tuple(t.shape)}")
    _check_out(smax_out, "smax_out", torch.float32, H)
    dev = _one_device([x, wqc, wkc, wqr, wkr, smax_out, workspace])
    B, S, D = x.shape
    if smax_out is None:
        smax_out = torch.empty(H, dtype=torch.float32, device=dev)
    need = int(lib.mc_mla_workspace_size(B, S, D, H, dc, dr))
    if need == 0:
        _check(lib.mc_mla_max_logit(None, None, None, None, None, B, S, D, H, dc, dr, int(causal), None, None, 0,
                                    None))
    with torch.cuda.device(dev):
        ws = workspace if workspace is not None else _workspace("mla", dev, need)
        _check(lib.mc_mla_max_logit(_ptr(x), _ptr(wqc), _ptr(wkc), _ptr(wqr), _ptr(wkr), B, S, D, H, dc, dr,
                                    int(causal), _ptr(smax_out), _ptr(ws), int(ws.numel() * ws.element_size()),
                                    _stream_handle(stream)))
    return smax_out


def polar_express_coeffs(steps: int = 10, l0: float = 1e-3, safety: float = 0.01):
    """Per-iteration (a, b, c) triples of a Polar Express schedule, for
    ``muon_step(..., ns_steps=steps, coeffs=...)`` (see mc_polar_express_coeffs).
    Host only."""
    lib = load_library()
    out = (ctypes.c_float * (3 * max(int(steps), 1)))()
    _check(lib.mc_polar_express_coeffs(int(steps), float(l0), float(safety), out))
    return [(float(out[3 * i]), float(out[3 * i + 1]), float(out[3 * i + 2])) for i in range(int(steps))]


def shard_plan(shapes, world: int, ns_steps: int = 5):
    """Owner rank of each (rows, cols) matrix and the per-rank Newton-Schulz
    cost (see mc_shard_plan).  Host only."""
    lib = load_library()
    n = len(shapes)
    rows = (ctypes.c_int64 * max(n, 1))(*[int(r) for r, _ in shapes])
    cols = (ctypes.c_int64 * max(n, 1))(*[int(c) for _, c in shapes])
    owner = (ctypes.c_int32 * max(n, 1))()
    load = (ctypes.c_double * max(world, 1))()
    _check(lib.mc_shard_plan(rows, cols, n, ns_steps, world, owner, load))
    return [int(owner[i]) for i in range(n)], [float(load[r]) for r in range(world)]


def qk_max_logit_static(x, wq, wk, H: int, dh: int, *, causal: bool = True, smax_out=None, stream=None):
    """S_max like ``qk_max_logit`` but through the allocation-free entry point
    (``mc_qk_max_logit_static``): no workspace is passed or allocated by the
    library; it uses its own fixed 64 MiB device scratch, limited to
    B*S*H*dh <= 2**24 and H <= 4096.  Calls that may overlap on the GPU race
    on that scratch.  (``smax_out`` is created here with torch if not given;
    pass it in to keep the whole call allocation-free.)"""
    torch = _torch()
    lib = load_library()
    _check_qk_args(x, wq, wk, H, dh, smax_out)
    dev = _one_device([x, wq, wk, smax_out])
    B, S, D = x.shape
    if smax_out is None:
        smax_out = torch.empty(H, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib.mc_qk_max_logit_static(_ptr(x), _ptr(wq), _ptr(wk), B, S, D, H, dh, int(causal),
                                          _ptr(smax_out), _stream_handle(stream)))
    return smax_out
