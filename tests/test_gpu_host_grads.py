"""GPU check of mc_muon_step_host_grads: with the gradients uploaded from
page-locked host memory piece by piece (overlapped with the step of the pieces
already there), every output equals mc_muon_step's bit for bit."""
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
SHAPES = [(256, 768), (768, 256), (512, 512), (300, 520), (520, 300), (64, 1000), (256, 768), (1000, 64),
          (128, 128), (512, 512)]


@pytest.mark.parametrize("chunks", [1, 3, 8, 50])
def test_host_grads_match_the_device_step(hp, chunks):
    mats = [wl.generic_matrix(r, c, seed=80 + i, g_dtype=(torch.float32 if i % 3 == 0 else torch.bfloat16))
            for i, (r, c) in enumerate(SHAPES)]

    def dev_copy():
        return ([W.to(DEV) for W, _, _ in mats], [M.to(DEV) for _, _, M in mats],
                [torch.empty(W.shape, dtype=torch.float32, device=DEV) for W, _, _ in mats],
                torch.zeros(len(mats), dtype=torch.float32, device=DEV))

    Wa, Ma, Ua, na = dev_copy()
    mc.muon_step(Wa, [G.to(DEV) for _, G, _ in mats], Ma, update_outs=Ua, norms_out=na, **hp)
    Wb, Mb, Ub, nb = dev_copy()
    g_host = [G.pin_memory() for _, G, _ in mats]
    g_dev = [torch.full(G.shape, float("nan"), dtype=G.dtype, device=DEV) for _, G, _ in mats]
    mc.muon_step_host_grads(Wb, g_dev, g_host, Mb, chunks=chunks, update_outs=Ub, norms_out=nb, **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    for a, b in zip(Wa + Ma + Ua + [na], Wb + Mb + Ub + [nb]):
        assert torch.equal(a.cpu(), b.cpu())
    for g, (_, G, _) in zip(g_dev, mats):
        assert torch.equal(g.cpu(), G)


def test_engine_owned_workspace_matches(hp):
    """NULL workspace (the library sizes and keeps its own) for mc_muon_step,
    mc_normuon_step and mc_muon_step_host_grads gives the results of the
    caller-workspace calls bit for bit."""
    import ctypes
    lib = mc.load_library()
    mats = [wl.generic_matrix(r, c, seed=90 + i) for i, (r, c) in enumerate(SHAPES[:6])]
    stream = torch.cuda.current_stream().cuda_stream

    def fresh():
        return ([W.to(DEV) for W, _, _ in mats], [G.to(DEV) for _, G, _ in mats], [M.to(DEV) for _, _, M in mats])

    # muon: binding (caller workspace) vs raw ABI call with NULL workspace
    Wa, Ga, Ma = fresh()
    mc.muon_step(Wa, Ga, Ma, **hp)
    Wb, Gb, Mb = fresh()
    arr, n = mc.make_params(Wb, Gb, Mb)
    h = mc.make_hparams(**hp)
    assert lib.mc_muon_step(arr, n, ctypes.byref(h), None, 0, None, stream) == mc.MC_OK, mc.last_error()
    # normuon, both ways
    Wc, Gc, Mc_ = fresh()
    Vc = [torch.zeros(W.shape[0], device=DEV) for W in Wc]
    mc.normuon_step(Wc, Gc, Mc_, Vc, **hp)
    Wd, Gd, Md = fresh()
    Vd = [torch.zeros(W.shape[0], device=DEV) for W in Wd]
    arr_d, _ = mc.make_params(Wd, Gd, Md)
    nm = mc.make_normuon(Vd)
    assert lib.mc_normuon_step(arr_d, n, ctypes.byref(h), ctypes.byref(nm), None, 0, None, stream) == mc.MC_OK
    # host grads with NULL workspace
    We, Ge, Me = fresh()
    keep = [G.pin_memory() for _, G, _ in mats]
    hptr = (ctypes.c_void_p * n)(*[k.data_ptr() for k in keep])
    arr_e, _ = mc.make_params(We, Ge, Me)
    assert lib.mc_muon_step_host_grads(arr_e, hptr, n, ctypes.byref(h), 3, None, 0, None, stream) == mc.MC_OK
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    for a, b, e in zip(Wa + Ma, Wb + Mb, We + Me):
        assert torch.equal(a.cpu(), b.cpu()) and torch.equal(a.cpu(), e.cpu())
    for a, b in zip(Wc + Mc_ + Vc, Wd + Md + Vd):
        assert torch.equal(a.cpu(), b.cpu())
