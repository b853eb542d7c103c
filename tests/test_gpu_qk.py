"""GPU parity of mc_qk_max_logit and mc_qk_clip (through the C ABI) against the
fp64 oracle: small ragged cases, a planted-score case that separates the causal
mask's two sides, and the full causal MHA layer (B 4, S 4096, H 32, dh 128)."""
import numpy as np
import pytest
import torch

import matrix_orthogonalising_optimizer_step_b200 as mc
import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
from gpu_util import GAMMA_TOL, SMAX_TOL, round_like, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_smax(X, Wq, Wk, H, dh, causal=True):
    s = mc.qk_max_logit(X.to(DEV), Wq.to(DEV), Wk.to(DEV), H, dh, causal=causal)
    assert mc.device_status() == mc.MC_OK, mc.last_error()
    return s.cpu().double().numpy()


def rel(a, b):
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-30)


# dh up to 256 takes the row-owned kernel (Q resident); dh = 320 (five 64-column
# k-blocks) the tile GEMM with the max epilogue
@pytest.mark.parametrize("B,S,D,H,dh", [(2, 300, 64, 3, 64), (1, 129, 40, 2, 72), (3, 700, 96, 4, 32),
                                        (1, 1, 16, 1, 8), (2, 520, 256, 2, 128), (1, 770, 64, 3, 256),
                                        (2, 333, 64, 2, 320), (1, 1300, 128, 5, 192)])
@pytest.mark.parametrize("causal", [True, False])
def test_smax_small(B, S, D, H, dh, causal):
    X, Wq, Wk = wl.qk_inputs(B, S, D, H, dh, seed=11, w_std=0.2)
    got = gpu_smax(X, Wq, Wk, H, dh, causal)
    ref = oracle.qk_max_logit(to64(X), to64(Wq), to64(Wk), H, dh, causal=causal)
    refb = oracle.qk_max_logit(to64(X), to64(Wq), to64(Wk), H, dh, causal=causal, qk_bf16=True)
    assert np.all(rel(got, ref) <= SMAX_TOL), (got, ref)
    # with Q and K rounded to bf16 as the kernel stores them, only accumulation
    # order and rare one-ulp rounding differences of Q/K remain
    assert np.all(rel(got, refb) <= 2e-3), (got, refb)


def test_planted_scores_respect_the_causal_mask():
    """q_517 . k_530 (j > i) is huge, q_530 . k_517 is its negative and the
    diagonals vanish: the causal max must stay at noise level while the
    unmasked max sees the planted pair."""
    B, S, D, H, dh = 1, 600, 64, 1, 64
    rng = np.random.default_rng(5)
    X = rng.normal(0, 0.01, (B, S, D))
    R = np.zeros((D, D))
    for k in range(D // 2):
        R[2 * k, 2 * k + 1] = -1.0
        R[2 * k + 1, 2 * k] = 1.0
    v = np.sign(rng.standard_normal(D))
    X[0, 517] = v
    X[0, 530] = R.T @ v
    Xt = wl.to_dtype(X, torch.bfloat16)
    Wq = wl.to_dtype(np.eye(D), torch.bfloat16)
    Wk = wl.to_dtype(R, torch.bfloat16)
    causal = gpu_smax(Xt, Wq, Wk, H, dh, True)
    full = gpu_smax(Xt, Wq, Wk, H, dh, False)
    assert full[0] == pytest.approx(D / np.sqrt(dh), rel=1e-2)
    assert causal[0] < 0.5
    ref = oracle.qk_max_logit(to64(Xt), to64(Wq), to64(Wk), H, dh, causal=True)
    assert abs(causal[0] - ref[0]) <= 1e-2 * max(abs(ref[0]), 1e-3) + 1e-4


def test_clip_small_against_oracle():
    H, dh, D = 4, 16, 64
    rng = np.random.default_rng(6)
    Wq = wl.to_dtype(rng.normal(0, 0.5, (H * dh, D)), torch.bfloat16)
    Wk = wl.to_dtype(rng.normal(0, 0.5, (H * dh, D)), torch.bfloat16)
    smax = torch.tensor([400.0, 80.0, 100.0, 250.0], dtype=torch.float32)
    q, k = Wq.to(DEV), Wk.to(DEV)
    gamma, mask = mc.qk_clip(q, k, smax.to(DEV), H, dh, tau=100.0, alpha=0.5)
    assert mc.device_status() == mc.MC_OK
    q, k, gamma, mask = q.cpu(), k.cpu(), gamma.cpu().double().numpy(), mask.cpu().numpy()
    oq, ok_, og, om = oracle.qk_clip(to64(Wq), to64(Wk), smax.double().numpy(), 100.0, 0.5, H, dh)
    assert list(mask) == list(om) == [1, 0, 0, 1]
    assert np.all(np.abs(gamma - og) <= GAMMA_TOL * og)
    assert gamma[0] == pytest.approx(0.25, abs=1e-7)
    for h in range(H):
        rows = slice(h * dh, (h + 1) * dh)
        if om[h]:
            # fp32 product rounded to bf16 vs the fp64 product rounded to bf16:
            # equal except where the two sit on either side of a rounding tie
            for got, want in ((q[rows], oq[rows]), (k[rows], ok_[rows])):
                g64, w64 = to64(got), round_like(want, torch.bfloat16)
                ulp = np.spacing(np.abs(w64).astype(np.float32)).astype(np.float64) * 65536
                assert np.all(np.abs(g64 - w64) <= ulp)
                assert np.mean(g64 == w64) >= 0.98
        else:
            assert torch.equal(q[rows], Wq[rows]) and torch.equal(k[rows], Wk[rows])


@pytest.fixture(scope="module")
def cfg3():
    X, Wq, Wk = wl.cfg3_inputs()
    c = wl.CFG3
    ref = oracle.qk_max_logit(to64(X), to64(Wq), to64(Wk), c["H"], c["dh"], causal=True)
    return X, Wq, Wk, ref


def test_cfg3_smax_and_clip(cfg3):
    X, Wq, Wk, ref = cfg3
    c = wl.CFG3
    H, dh = c["H"], c["dh"]
    x, q, k = X.to(DEV), Wq.to(DEV), Wk.to(DEV)
    smax = mc.qk_max_logit(x, q, k, H, dh, causal=True)
    assert mc.device_status() == mc.MC_OK
    got = smax.cpu().double().numpy()
    assert np.all(rel(got, ref) <= SMAX_TOL), np.max(rel(got, ref))
    gamma, mask = mc.qk_clip(q, k, smax, H, dh, tau=wl.QK_TAU, alpha=wl.QK_ALPHA)
    _, _, og, om = oracle.qk_clip(to64(Wq), to64(Wk), ref, wl.QK_TAU, wl.QK_ALPHA, H, dh)
    mask = mask.cpu().numpy()
    assert sorted(np.nonzero(mask)[0].tolist()) == sorted(np.nonzero(om)[0].tolist()) == list(c["hot_heads"])
    assert np.all(np.abs(gamma.cpu().double().numpy() - og) <= GAMMA_TOL * og)
    qc, kc = q.cpu(), k.cpu()
    for h in range(H):
        rows = slice(h * dh, (h + 1) * dh)
        if not mask[h]:
            assert torch.equal(qc[rows], Wq[rows]) and torch.equal(kc[rows], Wk[rows])
    # the clipped heads come back to tau (bf16 weights: within 2^-7)
    after = mc.qk_max_logit(x, q, k, H, dh, causal=True).cpu().double().numpy()
    for h in c["hot_heads"]:
        assert after[h] <= wl.QK_TAU * (1 + 2 ** -7)
        assert after[h] >= wl.QK_TAU * (1 - 2 ** -6)
    for h in range(H):
        if not mask[h]:
            assert after[h] == got[h]


@pytest.mark.parametrize("H", [4096, 4100])
def test_many_heads_both_sides_of_the_shared_head_table(H):
    """The causal max keeps per-head maxima in shared memory for up to 4096
    heads and uses global atomics beyond: both sides against the oracle."""
    B, S, D, dh = 1, 40, 16, 8
    X, Wq, Wk = wl.qk_inputs(B, S, D, H, dh, seed=19, w_std=0.3)
    got = gpu_smax(X, Wq, Wk, H, dh)
    refb = oracle.qk_max_logit(to64(X), to64(Wq), to64(Wk), H, dh, causal=True, qk_bf16=True)
    assert np.all(rel(got, refb) <= 2e-3), np.max(rel(got, refb))


def test_binding_rejects_mismatched_shapes_before_the_call():
    """The C side builds its tensor maps from H*dh and D, so a W_q or W_k with
    too few rows, or a too-short output, must be refused before any launch."""
    B, S, D, H, dh = 1, 64, 64, 2, 64
    X, Wq, Wk = wl.qk_inputs(B, S, D, H, dh, seed=5)
    x, wq, wk = X.to("cuda"), Wq.to("cuda"), Wk.to("cuda")
    short = wq[: H * dh - 8].contiguous()
    for fn in (mc.qk_max_logit, mc.qk_max_logit_static):
        with pytest.raises(ValueError):
            fn(x, short, wk, H, dh)
        with pytest.raises(ValueError):
            fn(x, wq, short, H, dh)
        with pytest.raises(ValueError):
            fn(x[0], wq, wk, H, dh)
        with pytest.raises(ValueError):
            fn(x, wq, wk, H, dh, smax_out=torch.zeros(H - 1, dtype=torch.float32, device="cuda"))
        with pytest.raises(TypeError):
            fn(x, wq, wk, H, dh, smax_out=torch.zeros(H, dtype=torch.float64, device="cuda"))
    with pytest.raises(ValueError):
        mc.qk_clip(short, short.clone(), torch.zeros(H, device="cuda"), H, dh)
    assert mc.device_status() == mc.MC_OK
