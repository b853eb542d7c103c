"""GPU parity of mc_muon_step (through the C ABI) against the fp64 oracle.

Element-by-element comparisons on small and ragged shapes that span several
128 x 256 tiles, every workload's shapes, and -- at the full 7B-shaped and MoE
sizes, in the same single call the benchmark times -- sampled matrices that
the oracle computes one by one."""
import numpy as np
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
from gpu_util import EW_TOL, NS_TOL, check_muon_matrix, rel_fro, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_step(mats, hp, update_mask=None):
    """mats: list of (W, G, M) CPU tensors.  Returns GPU results on the CPU."""
    Ws = [W.to(DEV).contiguous() for W, _, _ in mats]
    Gs = [G.to(DEV).contiguous() for _, G, _ in mats]
    Ms = [M.to(DEV).contiguous() for _, _, M in mats]
    Us = [torch.full(W.shape, float("nan"), dtype=torch.float32, device=DEV)
          if (update_mask is None or update_mask[i]) else None for i, (W, _, _) in enumerate(mats)]
    norms = torch.zeros(len(mats), dtype=torch.float32, device=DEV)
    mc.muon_step(Ws, Gs, Ms, norms_out=norms, update_outs=Us, **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    return ([W.cpu() for W in Ws], [M.cpu() for M in Ms],
            [U.cpu() if U is not None else None for U in Us], norms.cpu())


def check_all(mats, hp, outs, tag):
    W1, M1, U1, nrm = outs
    errs = []
    for i, (W0, G, M0) in enumerate(mats):
        ref = oracle.muon_step(to64(W0), to64(G), to64(M0), **hp)
        errs.append(check_muon_matrix(W0, G, M0, W1[i], M1[i], U1[i], nrm[i], hp, ref, f"{tag}[{i}]"))
    return errs


def test_cfg0_single_fp32_matrix(hp):
    mats = [wl.cfg0_matrix()]
    errs = check_all(mats, hp, run_step(mats, hp), "cfg0")
    assert errs[0][0] < 1e-2


@pytest.mark.parametrize("nesterov,ns_steps", [(True, 1), (False, 5), (True, 7)])
def test_hparam_variants(hp, nesterov, ns_steps):
    h = dict(hp, nesterov=nesterov, ns_steps=ns_steps)
    mats = [wl.generic_matrix(200, 330, seed=1), wl.generic_matrix(330, 200, seed=2)]
    check_all(mats, h, run_step(mats, h), f"nest{nesterov}-ns{ns_steps}")


CUBIC = (1.5, -0.5, 0.0)          # "Muon and MuonClip: orthogonalised updates for LLM training", §2
SIMPLE = (2.0, -1.5, 0.5)
TUNED = (3.4445, -4.7750, 2.0315)


@pytest.mark.parametrize("name,sched", [
    ("cubic x12", [CUBIC] * 12),
    ("simple quintic x8", [SIMPLE] * 8),
    ("tuned x3 then simple x4", [TUNED] * 3 + [SIMPLE] * 4),
])
def test_coefficient_schedules(hp, name, sched):
    h = dict(hp, ns_steps=len(sched), coeffs=sched)
    mats = [wl.generic_matrix(256, 768, seed=31), wl.generic_matrix(768, 256, seed=32),
            wl.cfg1_matrix(0, n=512)]
    check_all(mats, h, run_step(mats, h), name)


def test_polar_express_schedule(hp):
    """Ten Polar Express steps (the library's own table) against the oracle
    running its own table: the first polynomial's slope of about 8 makes the
    first two iterations the hardest for bf16 operands."""
    sched = mc.polar_express_coeffs(10)
    ref_sched = oracle.polar_express_schedule(10)
    h = dict(hp, ns_steps=10, coeffs=sched)
    h_ref = dict(hp, ns_steps=10, coeffs=ref_sched)
    mats = [wl.generic_matrix(256, 768, seed=33), wl.generic_matrix(768, 256, seed=34), wl.cfg1_matrix(1, n=512)]
    W1, M1, U1, nrm = run_step(mats, h)
    for i, (W0, G, M0) in enumerate(mats):
        ref = oracle.muon_step(to64(W0), to64(G), to64(M0), **h_ref)
        check_muon_matrix(W0, G, M0, W1[i], M1[i], U1[i], nrm[i], h_ref, ref, f"polar express[{i}]")


RAGGED = [(1, 1), (3, 5), (5, 3), (8, 1), (64, 64), (100, 37), (37, 100), (129, 129),
          (256, 256), (300, 520), (520, 300), (129, 1000), (1000, 129), (640, 384)]


def test_ragged_and_tall_wide_shapes(hp):
    mats = [wl.generic_matrix(r, c, seed=i) for i, (r, c) in enumerate(RAGGED)]
    check_all(mats, hp, run_step(mats, hp), "ragged")


THIN = [(2, 70000), (70000, 2), (32, 1024), (1024, 32), (12, 1025), (1025, 12), (16, 16), (32, 32),
        (31, 33), (33, 31)]


def test_thin_matrices_and_the_tensor_core_boundary(hp):
    """Short side <= 32: the fp32 thin path (several 256-column chunks, a
    chunk boundary, both orientations), in one call beside matrices just past
    the boundary that take the tensor-core GEMMs."""
    shapes = THIN + [(33, 90), (90, 33), (48, 48)]
    mats = [wl.generic_matrix(r, c, seed=500 + i) for i, (r, c) in enumerate(shapes)]
    mats.append(wl.generic_matrix(24, 700, seed=600, w_dtype=torch.float32, g_dtype=torch.float32))
    errs = check_all(mats, hp, run_step(mats, hp), "thin")
    # the thin path is fp32 throughout: far inside the bound
    for (r, c), e in zip(shapes, errs):
        if min(r, c) <= 32:
            assert e[0] < 1e-4, ((r, c), e[0])


def test_mixed_dtypes_and_repeated_shapes(hp):
    f32, bf = torch.float32, torch.bfloat16
    mats = []
    for i in range(3):
        mats.append(wl.generic_matrix(192, 320, seed=100 + i))
        mats.append(wl.generic_matrix(320, 192, seed=200 + i, w_dtype=f32))
        mats.append(wl.generic_matrix(256, 256, seed=300 + i, g_dtype=f32))
    # more than four shape groups -> several grouped launches per phase
    mats += [wl.generic_matrix(64 + 8 * k, 72, seed=400 + k) for k in range(6)]
    check_all(mats, hp, run_step(mats, hp), "mixed")


def test_zero_gradient_and_momentum_give_pure_decay(hp):
    r, c = 96, 160
    W = wl.to_dtype(np.random.default_rng(0).normal(0, 0.02, (r, c)), torch.bfloat16)
    mats = [(W, torch.zeros((r, c), dtype=torch.bfloat16), torch.zeros((r, c), dtype=torch.float32))]
    W1, M1, U1, nrm = run_step(mats, hp)
    assert float(nrm[0]) == 0.0
    assert torch.count_nonzero(U1[0]) == 0
    want = wl.to_dtype(to64(W) * (1 - hp["lr"] * hp["wd"]), torch.bfloat16)
    assert torch.equal(W1[0], want)


def test_transpose_symmetry(hp):
    """G and G^T take different kernel paths (MN-major Gram vs K-major); the
    updates must be transposes of each other to bf16 accuracy."""
    W, G, M = wl.generic_matrix(384, 1280, seed=7)
    mats = [(W, G, M), (W.T.contiguous(), G.T.contiguous(), M.T.contiguous())]
    _, _, U1, _ = run_step(mats, hp)
    assert rel_fro(to64(U1[1]).T, to64(U1[0])) <= 1e-2


def test_deterministic_bitwise(hp):
    mats = [wl.generic_matrix(512, 768, seed=s) for s in range(3)] + [wl.generic_matrix(768, 512, seed=9)]
    a = run_step(mats, hp)
    b = run_step(mats, hp)
    for x, y in zip(a[0] + a[1] + a[2], b[0] + b[1] + b[2]):
        assert torch.equal(x, y)
    assert torch.equal(a[3], b[3])


def test_cfg1_64_square_matrices(hp):
    mats = [wl.cfg1_matrix(i) for i in range(64)]
    errs = check_all(mats, hp, run_step(mats, hp), "cfg1")
    worst = max(e[0] for e in errs)
    assert worst <= NS_TOL
    print(f"cfg1 worst update rel err {worst:.3e}")


def _full_size_sampled(hp, shapes, sample_idx, host_matrix, device_gen):
    """Run one Muon step over the full list of `shapes` (device-drawn inputs)
    with the sampled indices replaced by host-drawn recipe matrices, then
    compare the sampled matrices against the oracle."""
    Ws, Gs, Ms = device_gen()
    host = {}
    for i in sample_idx:
        W, G, M = host_matrix(i)
        host[i] = (W, G, M)
        Ws[i].copy_(W.to(DEV)); Gs[i].copy_(G.to(DEV)); Ms[i].copy_(M.to(DEV))
    Us = [torch.empty(s, dtype=torch.float32, device=DEV) if i in host else None for i, s in enumerate(shapes)]
    norms = torch.zeros(len(shapes), dtype=torch.float32, device=DEV)
    mc.muon_step(Ws, Gs, Ms, norms_out=norms, update_outs=Us, **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    out = {}
    for i in sample_idx:
        out[i] = (Ws[i].cpu(), Ms[i].cpu(), Us[i].cpu(), norms[i].cpu())
    del Ws, Gs, Ms, Us
    mc.release_workspaces()
    torch.cuda.empty_cache()
    for i in sample_idx:
        W0, G, M0 = host[i]
        ref = oracle.muon_step(to64(W0), to64(G), to64(M0), **hp)
        e = check_muon_matrix(W0, G, M0, *out[i], hp, ref, f"sample[{i}]")
        print(f"sample {i} {tuple(W0.shape)}: update rel err {e[0]:.3e}, dW rel err {e[1]:.3e}")


def test_cfg2_full_size_sampled(hp):
    shapes = wl.cfg2_shapes()
    _full_size_sampled(hp, shapes, [0, 4, 6, 223], wl.cfg2_matrix,
                       lambda: wl.cfg2_device_tensors(DEV))


def test_cfg4_full_size_sampled(hp):
    shapes = wl.cfg4_shapes()

    def gen():
        g = torch.Generator(device=DEV)
        g.manual_seed(4004)
        Ws = [(torch.randn(s, device=DEV, generator=g) * 0.02).to(torch.bfloat16) for s in shapes]
        Gs = [(torch.randn(s, device=DEV, generator=g) * 1e-3).to(torch.bfloat16) for s in shapes]
        Ms = [torch.zeros(s, device=DEV, dtype=torch.float32) for s in shapes]
        return Ws, Gs, Ms
    _full_size_sampled(hp, shapes, [0, 2, 191], wl.cfg4_matrix, gen)


@pytest.mark.parametrize("r,c", [(32768, 65600), (65600, 32768)])
def test_matrix_past_2_31_elements(hp, r, c):
    """One 2.15e9-element weight (past 2^31), wide and tall: 64-bit indexing
    in the momentum kernel, the GEMM epilogues and the apply.  The oracle
    cannot run at this size, so the checks are elementwise on sampled flat
    indices (momentum; the apply against the update it reports) and, for the
    Newton-Schulz output O, properties that hold at any size: O X0^T (tall:
    X0^T O) is symmetric (O = q(X0 X0^T) X0 for the composed polynomial q),
    and the singular values sit near the polynomial's band, so
    ||O||_F / sqrt(min(r, c)) does."""
    g = torch.Generator(device=DEV)
    g.manual_seed(123)
    W = (torch.randn((r, c), device=DEV, generator=g) * 0.02).to(torch.bfloat16)
    G = (torch.randn((r, c), device=DEV, generator=g) * 1e-3).to(torch.bfloat16)
    M = torch.randn((r, c), device=DEV, generator=g) * 1e-3
    idx = torch.cat([torch.randint(0, r * c, (4000,), device=DEV, generator=g),
                     torch.tensor([0, 2**31 - 1, 2**31, 2**31 + 12345, r * c - 1], device=DEV)])
    w0, g0, m0 = W.view(-1)[idx].double().cpu(), G.view(-1)[idx].double().cpu(), M.view(-1)[idx].double().cpu()
    mu = float(np.float32(hp["mu"]))
    # the NS input, kept for the property check (fp32, the kernels' own arithmetic)
    m_new = torch.addcmul(G.float(), M, torch.tensor(mu, device=DEV))
    X0 = G.float() + mu * m_new if hp["nesterov"] else m_new.clone()
    del m_new
    X0 /= torch.linalg.vector_norm(X0)
    U = torch.empty((r, c), dtype=torch.float32, device=DEV)
    mc.muon_step([W], [G], [M], update_outs=[U], **hp)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    # momentum, elementwise
    m1 = M.view(-1)[idx].double().cpu()
    want = mu * m0 + g0
    assert torch.all(torch.abs(m1 - want) <= 1e-6 * torch.abs(want) + 1e-12)
    # the apply: W1 = (1 - lr wd) W0 - lr U, to one bf16 ulp
    w1, u = W.view(-1)[idx].double().cpu(), U.view(-1)[idx].double().cpu()
    w_exp = (1 - hp["lr"] * hp["wd"]) * w0 - hp["lr"] * u
    ulp = torch.from_numpy(np.spacing(np.abs(w_exp.numpy()).astype(np.float32)).astype(np.float64)) * 65536
    assert torch.all(torch.abs(w1 - w_exp) <= ulp)
    # Newton-Schulz output O = U / (rms * sqrt(max(r, c)))
    O = U / (hp["rms_scale"] * np.sqrt(max(r, c)))
    del U
    # A Gaussian X0 of this shape has its singular values in [1.6e-3, 9.4e-3]
    # (Marchenko-Pastur edges over ||X0||_F); five tuned quintic steps map them
    # into [0.68, 1.20], and weighting by the Marchenko-Pastur density gives
    # ||O||_F / sqrt(m) = 1.020 in exact arithmetic.
    scale = float(torch.linalg.vector_norm(O)) / np.sqrt(min(r, c))
    assert abs(scale - 1.020) <= 0.04, scale
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        P = X0.T @ O if r > c else O @ X0.T
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    asym = float(torch.linalg.matrix_norm(P - P.T) / torch.linalg.matrix_norm(P))
    assert asym <= 2e-2, asym
    print(f"2^31+ matrix {r}x{c}: ||O||_F/sqrt(m) = {scale:.3f}, asymmetry = {asym:.2e}")
    del W, G, M, X0, O, P
    mc.release_workspaces()
    torch.cuda.empty_cache()


def test_many_matrices_tables_in_several_launches(hp):
    """Four hundred small matrices in one call: their parameter tables (about
    38 KB) go up in two table launches (32704 bytes of parameters at most per
    launch).  Every matrix is checked against the oracle."""
    shapes = [(64, 96), (96, 64), (48, 80), (128, 128)]
    mats = [wl.generic_matrix(*shapes[i % 4], seed=1000 + i) for i in range(400)]
    mc.profile_begin()
    outs = run_step(mats, hp)
    k = mc.profile_end()
    assert k["table_upload"]["launches"] == 2, k["table_upload"]
    check_all(mats, hp, outs, "many")
