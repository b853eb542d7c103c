"""GPU parity of mc_normuon_step (through the C ABI) against the fp64 oracle:
the Muon step with NorMuon's per-row normalisation ("About Muon: Muon At
Scale", "Certain Neurons Still Dominate").  Wide, tall, square and ragged
shapes; bf16 and fp32 weights; rows whose length is not a multiple of 8; the
row state carried over two steps; and the 7B-shaped set at full size on
sampled matrices."""
import numpy as np
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
from gpu_util import EW_TOL, NS_TOL, check_muon_matrix, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
BETA2, EPS_V = 0.95, 1e-8


def _row_scaled(r, c, seed, w_dtype=torch.bfloat16):
    """Gradients whose rows differ in scale (so the row pass has work to do)."""
    rng = wl.rng_for(95, seed, r, c)
    W = wl.to_dtype(rng.normal(0, 0.02, (r, c)), w_dtype)
    G = wl.to_dtype(rng.normal(0, 1e-3, (r, c)) * np.exp(rng.normal(0, 1, (r, 1))), torch.bfloat16)
    M = wl.to_dtype(rng.normal(0, 1e-3, (r, c)), torch.float32)
    v = torch.from_numpy(np.abs(rng.normal(0, 1e-3, r))).to(torch.float32)
    return W, G, M, v


def _run(mats, hp, steps=1):
    Ws = [W.to(DEV) for W, _, _, _ in mats]
    Gs = [G.to(DEV) for _, G, _, _ in mats]
    Ms = [M.to(DEV) for _, _, M, _ in mats]
    Vs = [v.to(DEV) for _, _, _, v in mats]
    Us = [torch.full(W.shape, float("nan"), dtype=torch.float32, device=DEV) for W in Ws]
    norms = torch.zeros(len(mats), dtype=torch.float32, device=DEV)
    for _ in range(steps):
        mc.normuon_step(Ws, Gs, Ms, Vs, beta2=BETA2, eps_v=EPS_V, norms_out=norms, update_outs=Us, **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    return [x.cpu() for x in Ws], [x.cpu() for x in Ms], [x.cpu() for x in Us], [x.cpu() for x in Vs], norms.cpu()


def _check(mats, hp, outs, tag):
    W1, M1, U1, V1, nrm = outs
    errs = []
    for i, (W0, G, M0, v0) in enumerate(mats):
        Wn, Mn, upd, vn = oracle.normuon_step(to64(W0), to64(G), to64(M0), to64(v0), beta2=BETA2, eps_v=EPS_V, **hp)
        norm = oracle.muon_step(to64(W0), to64(G), to64(M0), **hp)[3]
        e = check_muon_matrix(W0, G, M0, W1[i], M1[i], U1[i], nrm[i], hp, (Wn, Mn, upd, norm), f"{tag}[{i}]")
        # the row state: the row mean squares of the NS output carry its error
        assert rel_fro(to64(V1[i]), vn) <= NS_TOL, f"{tag}[{i}] v"
        # NorMuon keeps the Frobenius norm of O: ||update|| = rms * ||O||_F
        errs.append(e)
    return errs


SHAPES = [(256, 768), (768, 256), (512, 512), (300, 520), (520, 300), (129, 1000), (1000, 129), (37, 100),
          (100, 37), (8, 1), (1, 8), (64, 64), (12, 1025), (1025, 12), (32, 600)]


def test_normuon_shapes_against_oracle(hp):
    mats = [_row_scaled(r, c, seed=i) for i, (r, c) in enumerate(SHAPES)]
    _check(mats, hp, _run(mats, hp), "normuon")


def test_normuon_fp32_weights_and_hparam_variants(hp):
    mats = [_row_scaled(200, 330, seed=50, w_dtype=torch.float32), _row_scaled(330, 200, seed=51),
            _row_scaled(96, 96, seed=52, w_dtype=torch.float32)]
    for h in (dict(hp, nesterov=False, ns_steps=1), dict(hp, ns_steps=2), dict(hp, ns_steps=7)):
        _check(mats, h, _run(mats, h), f"ns{h['ns_steps']}")


def test_normuon_state_over_two_steps(hp):
    """The second step uses the first step's row state and momentum."""
    mats = [_row_scaled(256, 384, seed=60), _row_scaled(384, 256, seed=61)]
    W1, M1, U1, V1, _ = _run(mats, hp, steps=2)
    for i, (W0, G, M0, v0) in enumerate(mats):
        w, m, v = to64(W0), to64(M0), to64(v0)
        for _ in range(2):
            w, m, upd, v = oracle.normuon_step(w, to64(G), m, v, beta2=BETA2, eps_v=EPS_V, **hp)
            w = to64(torch.from_numpy(w).to(W0.dtype))     # the weight is stored in its dtype between steps
        assert rel_fro(to64(M1[i]), m) <= EW_TOL
        assert rel_fro(to64(U1[i]), upd) <= NS_TOL
        assert rel_fro(to64(V1[i]), v) <= NS_TOL
        assert rel_fro(to64(W1[i]) - to64(W0), w - to64(W0)) <= 2 * NS_TOL


def test_normuon_with_frozen_state_matches_muon(hp):
    """A huge, uniform row state makes the row division uniform (v ~ beta2 *
    1e6 on every row), so NorMuon's update equals Muon's up to the NS error of
    each path (their NS kernels are the same)."""
    mats = [_row_scaled(256, 512, seed=70), _row_scaled(512, 256, seed=71)]
    big = [(W, G, M, torch.full((W.shape[0],), 1e6)) for W, G, M, _ in mats]
    _, _, Un, _, _ = _run(big, hp)
    Ws = [W.to(DEV) for W, _, _, _ in mats]
    Gs = [G.to(DEV) for _, G, _, _ in mats]
    Ms = [M.to(DEV) for _, _, M, _ in mats]
    Us = [torch.empty(W.shape, dtype=torch.float32, device=DEV) for W in Ws]
    mc.muon_step(Ws, Gs, Ms, update_outs=Us, **hp)
    for a, b in zip(Un, Us):
        assert rel_fro(to64(a), to64(b.cpu())) <= 1e-5


def test_normuon_7b_full_size_sampled(hp):
    """The whole 7B-shaped set in one call (as a NorMuon step would run it),
    with sampled matrices drawn on the host and checked against the oracle."""
    shapes = wl.cfg2_shapes()
    Ws, Gs, Ms = wl.cfg2_device_tensors(DEV)
    Vs = [torch.zeros(s[0], dtype=torch.float32, device=DEV) for s in shapes]
    sample = [0, 4, 6, 223]
    host = {}
    for i in sample:
        W, G, M = wl.cfg2_matrix(i)
        host[i] = (W, G, M)
        Ws[i].copy_(W.to(DEV)); Gs[i].copy_(G.to(DEV)); Ms[i].copy_(M.to(DEV))
    Us = [torch.empty(s, dtype=torch.float32, device=DEV) if i in host else None for i, s in enumerate(shapes)]
    norms = torch.zeros(len(shapes), dtype=torch.float32, device=DEV)
    mc.normuon_step(Ws, Gs, Ms, Vs, beta2=BETA2, eps_v=EPS_V, norms_out=norms, update_outs=Us, **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    out = {i: (Ws[i].cpu(), Ms[i].cpu(), Us[i].cpu(), Vs[i].cpu(), norms[i].cpu()) for i in sample}
    del Ws, Gs, Ms, Us, Vs
    mc.release_workspaces()
    torch.cuda.empty_cache()
    for i in sample:
        W0, G, M0 = host[i]
        v0 = torch.zeros(W0.shape[0], dtype=torch.float32)
        Wn, Mn, upd, vn = oracle.normuon_step(to64(W0), to64(G), to64(M0), to64(v0), beta2=BETA2, eps_v=EPS_V, **hp)
        norm = oracle.muon_step(to64(W0), to64(G), to64(M0), **hp)[3]
        W1, M1, U1, V1, n1 = out[i]
        e = check_muon_matrix(W0, G, M0, W1, M1, U1, n1, hp, (Wn, Mn, upd, norm), f"sample[{i}]")
        assert rel_fro(to64(V1), vn) <= NS_TOL
        print(f"normuon sample {i} {tuple(W0.shape)}: update rel err {e[0]:.3e}")
