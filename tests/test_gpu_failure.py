"""Failure detection on the GPU, without faulting, trapping or hanging it.

* A bounded wait that runs out: every wait in the library's kernels gives up
  after a limit instead of spinning forever, raises the device error word and
  lets the kernel return.  mc_selftest_bounded_wait makes one such wait (on an
  mbarrier nothing arrives on) run out after a short limit; the status must
  read MC_ERR_DEVICE once, then MC_OK, and the next real call must be right.
* Non-finite input ("MuonClip: speed, then stability" §12 lists overflow
  events among what a run should watch): a NaN or Inf in one matrix's
  gradient or momentum is reported (its norms_out entry is not finite, the
  status reads MC_ERR_NONFINITE) and contained: that matrix's W only decays,
  and the other matrices of the call are exactly as without it.
"""
import numpy as np
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
from gpu_util import check_muon_matrix, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _step(mats, hp):
    Ws = [W.to(DEV) for W, _, _ in mats]
    Gs = [G.to(DEV) for _, G, _ in mats]
    Ms = [M.to(DEV) for _, _, M in mats]
    Us = [torch.empty(W.shape, dtype=torch.float32, device=DEV) for W in Ws]
    norms = torch.zeros(len(mats), dtype=torch.float32, device=DEV)
    mc.muon_step(Ws, Gs, Ms, norms_out=norms, update_outs=Us, **hp)
    return Ws, Ms, Us, norms


def test_bounded_wait_runs_out_and_the_context_stays_usable(hp):
    lib = mc.load_library()
    assert mc.device_status() == mc.MC_OK
    rc = lib.mc_selftest_bounded_wait(2_000_000, torch.cuda.current_stream().cuda_stream)
    assert rc == mc.MC_OK, mc.last_error()
    assert mc.device_status() == mc.MC_ERR_DEVICE
    assert "bounded wait" in mc.last_error()
    assert mc.device_status() == mc.MC_OK          # read and cleared
    mats = [wl.generic_matrix(200, 330, seed=71), wl.generic_matrix(12, 900, seed=72)]
    Ws, Ms, Us, norms = _step(mats, hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    for i, (W0, G, M0) in enumerate(mats):
        ref = oracle.muon_step(to64(W0), to64(G), to64(M0), **hp)
        check_muon_matrix(W0, G, M0, Ws[i].cpu(), Ms[i].cpu(), Us[i].cpu(), norms[i].cpu(), hp, ref, f"after[{i}]")


def test_non_finite_gradient_is_reported_and_contained(hp):
    clean = [wl.generic_matrix(330, 200, seed=81), wl.generic_matrix(256, 256, seed=82),
             wl.generic_matrix(20, 700, seed=83)]
    bad_nan = wl.generic_matrix(200, 330, seed=84)   # tensor-core path, NaN in G
    bad_inf = wl.generic_matrix(8, 600, seed=85)     # thin path, Inf in M
    bad_nan[1][17, 5] = float("nan")
    bad_inf[2][3, 400] = float("inf")
    mats = [bad_nan, clean[0], bad_inf, clean[1], clean[2]]
    Ws, Ms, Us, norms = _step(mats, hp)
    assert mc.device_status() == mc.MC_ERR_NONFINITE
    assert "non-finite" in mc.last_error()
    assert mc.device_status() == mc.MC_OK
    nrm = norms.cpu()
    assert torch.isnan(nrm[0]) and torch.isinf(nrm[2])
    for i in (0, 2):
        W0 = mats[i][0]
        assert torch.count_nonzero(Us[i].cpu()) == 0
        want = wl.to_dtype(to64(W0) * (1 - hp["lr"] * hp["wd"]), W0.dtype)
        assert torch.equal(Ws[i].cpu(), want)
    # the other matrices: as the oracle, and bit for bit as in a call without the bad ones
    Wc, Mc, Uc, nc = _step(clean, hp)
    assert mc.device_status() == mc.MC_OK
    for j, i in enumerate((1, 3, 4)):
        W0, G, M0 = mats[i]
        ref = oracle.muon_step(to64(W0), to64(G), to64(M0), **hp)
        check_muon_matrix(W0, G, M0, Ws[i].cpu(), Ms[i].cpu(), Us[i].cpu(), nrm[i], hp, ref, f"clean[{i}]")
        assert torch.equal(Ws[i].cpu(), Wc[j].cpu())
        assert torch.equal(Us[i].cpu(), Uc[j].cpu())
