"""Pins for the fp64 oracle: each test ties an oracle function to something
other than itself -- the odd-polynomial/SVD identity, numbers the pages print
(tests/golden/printed_numbers.json, each entry cited), brute force on tiny
inputs, limits with a textbook answer, or a third-party optimizer run as a
library.  CPU only."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from matrix_orthogonalising_optimizer_step_b200 import workloads as wl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "printed_numbers.json")))
TUNED = tuple(GOLD["tuned_coefficients"]["value"])


def haar(rng, n, k):
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


# ---------------------------------------------------------------- scalar map
def test_scalar_map_printed_properties():
    a, b, c = GOLD["simple_quintic"]["value"]
    assert oracle.phi(1.0, a, b, c) == pytest.approx(GOLD["simple_quintic"]["phi_at_1"], abs=1e-15)
    h = 1e-6
    d = (oracle.phi(1 + h, a, b, c) - oracle.phi(1 - h, a, b, c)) / (2 * h)
    assert d == pytest.approx(GOLD["simple_quintic"]["dphi_at_1"], abs=1e-8)
    a3, b3, c3 = GOLD["classic_cubic"]["value"]
    # The cubic converges to exactly 1 from inside (0, 1].
    assert oracle.phi_iter(0.3, 60, a3, b3, c3) == pytest.approx(1.0, abs=1e-12)


def test_scalar_map_polar_express_number():
    g = GOLD["polar_express_vs_ns"]
    y = oracle.phi_iter(g["x0"], g["steps"], *TUNED)
    assert abs(y - g["printed"]) <= g["tol"]


def test_scalar_map_overshoot_and_band():
    xs = np.linspace(1e-6, 1.0, 400_001)
    y = oracle.phi_iter(xs, 5, *TUNED)
    g = GOLD["tuned_overshoot_max"]
    assert abs(y.max() - g["printed"]) <= g["tol"]
    band = GOLD["tuned_band"]
    sel = xs >= band["x_from"]
    assert y[sel].min() >= band["lo"] - band["slack"]
    assert y[sel].max() <= band["hi"] + band["slack"]
    jb = GOLD["jordan_band"]
    assert jb["lo"] - 0.02 <= y[sel].min() and y.max() <= jb["hi"]


def test_scalar_map_demo_numbers_are_consistent():
    from scipy.optimize import brentq
    g = GOLD["demo_consistency"]
    x0 = brentq(lambda x: oracle.phi_iter(x, 5, *TUNED) - g["tuned_5"], 1e-5, 1e-2)
    simple = tuple(GOLD["simple_quintic"]["value"])
    assert abs(oracle.phi_iter(x0, 5, *simple) - g["simple_5"]) <= g["tol_simple_5"]
    assert abs(oracle.phi_iter(x0, 10, *simple) - g["simple_10"]) <= g["tol_simple_10"]


# ---------------------------------------------------------- matrix iteration
@pytest.mark.parametrize("shape", [(24, 40), (40, 24), (32, 32), (7, 19)])
def test_ns_equals_scalar_map_on_singular_values(shape):
    """Odd-polynomial identity: NS(U diag(s) V^T) = U diag(phi^N(s/||s||)) V^T."""
    r, c = shape
    m = min(r, c)
    rng = np.random.default_rng(11 + r * 100 + c)
    U, V = haar(rng, r, m), haar(rng, c, m)
    s = np.sort(rng.uniform(0.01, 3.0, m))[::-1]
    G = (U * s) @ V.T
    want = (U * oracle.phi_iter(s / np.linalg.norm(s), 5, *TUNED)) @ V.T
    got = oracle.newton_schulz(G, 5, *TUNED)
    assert np.linalg.norm(got - want) <= 1e-12 * np.linalg.norm(want)


def test_ns_on_diagonal_is_scalar_map_entrywise():
    d = np.array([3.0, -1.0, 0.5, 0.02, 0.0])
    G = np.zeros((5, 9))
    G[np.arange(5), np.arange(5)] = d
    got = oracle.newton_schulz(G, 5, *TUNED)
    want = np.zeros_like(G)
    want[np.arange(5), np.arange(5)] = oracle.phi_iter(d / np.linalg.norm(d), 5, *TUNED)
    assert np.max(np.abs(got - want)) <= 1e-14


def test_ns_keeps_singular_vectors_and_band_and_approaches_polar():
    rng = np.random.default_rng(5)
    r, c = 48, 80
    U, V = haar(rng, r, r), haar(rng, c, r)
    s = np.linspace(1.0, 0.1, r)
    G = (U * s) @ V.T
    O = oracle.newton_schulz(G, 5, *TUNED)
    D = U.T @ O @ V
    off = D - np.diag(np.diag(D))
    assert np.max(np.abs(off)) <= 1e-10
    sv = np.diag(D)
    assert sv.min() >= 0.68 and sv.max() <= 1.21
    P = U @ V.T
    assert np.linalg.norm(O - P) / np.linalg.norm(P) <= 0.32


def test_ns_converges_to_svd_polar_factor_with_simple_quintic():
    """With phi(1) = 1, phi'(1) = 0 the iteration converges to U V^T, the
    polar factor that numpy's SVD gives (textbook limit)."""
    rng = np.random.default_rng(6)
    G = rng.standard_normal((30, 50)) + 3 * np.eye(30, 50)
    u, _, vt = np.linalg.svd(G, full_matrices=False)
    O = oracle.newton_schulz(G, 40, *GOLD["simple_quintic"]["value"])
    assert np.linalg.norm(O - u @ vt) <= 1e-9 * np.linalg.norm(u @ vt)


def test_ns_orientation_transpose_equivariant():
    rng = np.random.default_rng(7)
    G = rng.standard_normal((20, 33))
    assert np.array_equal(oracle.newton_schulz(G.T, 5, *TUNED), oracle.newton_schulz(G, 5, *TUNED).T)


def test_ns_zero_matrix_gives_zero():
    assert np.array_equal(oracle.newton_schulz(np.zeros((4, 6)), 5, *TUNED), np.zeros((4, 6)))


# ----------------------------------------------------------------- the step
def test_update_rms_is_point_two_for_exact_polar_factor(hp):
    """0.2 sqrt(max(m,n)) U V^T has entry RMS exactly 0.2 (printed target).
    Uses the converging simple quintic so that NS reaches U V^T."""
    rng = np.random.default_rng(8)
    for (r, c) in [(40, 90), (90, 40), (64, 64)]:
        G = rng.standard_normal((r, c)) + 2 * np.eye(r, c)
        p = dict(hp, ns_steps=40, a=2.0, b=-1.5, c=0.5, lr=1.0, wd=0.0, mu=0.0, nesterov=False)
        _, _, upd, _ = oracle.muon_step(np.zeros((r, c)), G, np.zeros((r, c)), **p)
        rms = np.sqrt(np.mean(upd ** 2))
        assert rms == pytest.approx(GOLD["rms_target"]["value"], rel=1e-10)


def test_update_rms_closed_form_for_tuned_ns(hp):
    """RMS of 0.2 sqrt(n) NS(G) = 0.2 sqrt(sum phi^5(s_i/||s||)^2 / m)."""
    rng = np.random.default_rng(9)
    r, c = 36, 100
    U, V = haar(rng, r, r), haar(rng, c, r)
    s = 1.0 / np.arange(1, r + 1)
    G = (U * s) @ V.T
    p = dict(hp, mu=0.0, nesterov=False)
    _, _, upd, _ = oracle.muon_step(np.zeros((r, c)), G, np.zeros((r, c)), **p)
    want = 0.2 * np.sqrt(np.sum(oracle.phi_iter(s / np.linalg.norm(s), 5, *TUNED) ** 2) / r)
    assert np.sqrt(np.mean(upd ** 2)) == pytest.approx(want, rel=1e-12)


def test_momentum_special_cases(hp):
    rng = np.random.default_rng(10)
    M0 = rng.standard_normal((6, 8))
    G = rng.standard_normal((6, 8))
    W = rng.standard_normal((6, 8))
    _, M1, _, _ = oracle.muon_step(W, np.zeros_like(G), M0, **hp)
    assert np.allclose(M1, hp["mu"] * M0, rtol=0, atol=0)
    _, M1, _, _ = oracle.muon_step(W, G, np.zeros_like(M0), **hp)
    assert np.array_equal(M1, G)


def test_nesterov_lookahead_diagonal_pin(hp):
    """With diagonal M0 = diag(p) and G = diag(q), Nesterov's NS input is
    diagonal (1+mu) q + mu^2 p, the plain one q + mu p; the update is then the
    scalar map on the normalised diagonal."""
    mu = hp["mu"]
    p_ = np.array([1.0, 0.2, 0.0, 0.05])
    q_ = np.array([0.0, 0.3, 0.7, 0.01])
    r, c = 4, 7
    M0 = np.zeros((r, c)); M0[range(4), range(4)] = p_
    G = np.zeros((r, c)); G[range(4), range(4)] = q_
    for nesterov, u in [(True, (1 + mu) * q_ + mu * mu * p_), (False, q_ + mu * p_)]:
        h = dict(hp, nesterov=nesterov)
        _, _, upd, nrm = oracle.muon_step(np.zeros((r, c)), G, M0, **h)
        want = np.zeros((r, c))
        want[range(4), range(4)] = 0.2 * np.sqrt(c) * oracle.phi_iter(u / np.linalg.norm(u), 5, *TUNED)
        assert np.max(np.abs(upd - want)) <= 1e-13
        assert nrm == pytest.approx(np.linalg.norm(u), rel=1e-14)


def test_first_step_independent_of_nesterov(hp):
    W, G, M = wl.cfg0_matrix()
    W, G, M = (t.double().numpy() for t in (W, G, M))
    a = oracle.muon_step(W, G, M, **dict(hp, nesterov=True))
    b = oracle.muon_step(W, G, M, **dict(hp, nesterov=False))
    assert np.max(np.abs(a[2] - b[2])) <= 1e-13 * np.max(np.abs(a[2]))


def test_decay_and_apply_special_cases(hp):
    rng = np.random.default_rng(12)
    W = rng.standard_normal((5, 9)); G = rng.standard_normal((5, 9)); M = rng.standard_normal((5, 9))
    Wn, _, _, _ = oracle.muon_step(W, G, M, **dict(hp, lr=0.0))
    assert np.array_equal(Wn, W)
    Wn, _, upd, _ = oracle.muon_step(W, G, M, **dict(hp, wd=0.0))
    assert np.allclose(Wn - W, -hp["lr"] * upd, rtol=1e-12, atol=1e-15)
    Wn, _, upd, _ = oracle.muon_step(W, np.zeros_like(G), np.zeros_like(M), **hp)
    assert np.array_equal(upd, np.zeros_like(upd))
    assert np.allclose(Wn, (1 - hp["lr"] * hp["wd"]) * W, rtol=1e-15, atol=0)


def test_cfg0_matches_torch_muon(hp):
    """Third-party run: torch.optim.Muon with Moonshot's RMS matching on the
    same cfg0 inputs (zero momentum, so its buffer convention does not matter
    after normalisation).  torch runs its NS in bf16 whatever the parameter
    dtype (measured: 2.08e-2 from this oracle with float32 and float64
    parameters alike; a bf16-rounding emulation of the oracle's own NS sits
    1.7e-2 away), so the bound is 3e-2.  It still separates the update scale
    0.2*sqrt(max) from 0.2*sqrt(min) (41 %) and a missing transpose."""
    W, G, M = wl.cfg0_matrix()
    p = torch.nn.Parameter(W.clone())
    opt = torch.optim.Muon([p], lr=hp["lr"], weight_decay=hp["wd"], momentum=hp["mu"],
                           nesterov=True, ns_coefficients=TUNED, eps=hp["eps"],
                           ns_steps=hp["ns_steps"], adjust_lr_fn="match_rms_adamw")
    p.grad = G.clone()
    opt.step()
    dW_t = (p.detach().double() - W.double()).numpy()
    Wn, _, _, _ = oracle.muon_step(W.double().numpy(), G.double().numpy(), M.double().numpy(), **hp)
    dW_o = Wn - W.double().numpy()
    assert np.linalg.norm(dW_t - dW_o) / np.linalg.norm(dW_o) <= 3e-2


# ----------------------------------------------------------------- QK-Clip
def test_smax_matches_bruteforce_and_planted_scores():
    rng = np.random.default_rng(13)
    B, S, D, H, dh = 2, 6, 5, 3, 2
    X = rng.standard_normal((B, S, D))
    Wq = rng.standard_normal((H * dh, D))
    Wk = rng.standard_normal((H * dh, D))
    for causal in (True, False):
        got = oracle.qk_max_logit(X, Wq, Wk, H, dh, causal=causal)
        want = oracle.qk_max_logit_bruteforce(X, Wq, Wk, H, dh, causal=causal)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-13)
    # Planted pair: a large score between query 1 and key 4 (j > i) must not
    # count under the causal mask; the same pair on the diagonal must count.
    X = np.zeros((1, 5, 2)); X[0, :, 1] = 0.01
    Wq = np.array([[1.0, 0.0], [0.0, 1.0]]); Wk = Wq.copy()
    X[0, 1, 0] = 10.0; X[0, 4, 0] = 10.0
    smax = oracle.qk_max_logit(X, Wq, Wk, 1, 2, causal=True)
    assert smax[0] == pytest.approx(oracle.qk_max_logit_bruteforce(X, Wq, Wk, 1, 2)[0])
    # query 4 sees key 4 (diagonal) -> 100.0001/sqrt(2); also query 4 sees key 1.
    assert smax[0] == pytest.approx((100.0 + 1e-4) / np.sqrt(2), rel=1e-12)
    X[0, 4, 0] = 0.0; X[0, 0, 0] = 10.0; X[0, 1, 0] = 0.0
    # now only query 0 / key 0 is large: the diagonal of row 0 counts.
    assert oracle.qk_max_logit(X, Wq, Wk, 1, 2)[0] == pytest.approx((100 + 1e-4) / np.sqrt(2), rel=1e-12)
    X[0, 0, 0] = 0.0; X[0, 0, 1] = 0.01; X[0, 3, 0] = 10.0; X[0, 2, 0] = -10.0
    # scores: q3.k3 = 100 counts; q2.k3 (j > i) = -100 would not anyway; signed max.
    assert oracle.qk_max_logit(X, Wq, Wk, 1, 2)[0] == pytest.approx((100 + 1e-4) / np.sqrt(2), rel=1e-12)


def test_smax_is_signed_max_not_abs():
    X = np.array([[[1.0], [1.0]]])
    Wq = np.array([[-3.0]]); Wk = np.array([[2.0]])
    assert oracle.qk_max_logit(X, Wq, Wk, 1, 1)[0] == pytest.approx(-6.0)


def test_clip_worked_example():
    g = GOLD["qk_clip_example"]
    H, dh, D = 2, 3, 4
    rng = np.random.default_rng(14)
    Wq = rng.standard_normal((H * dh, D)); Wk = rng.standard_normal((H * dh, D))
    smax = np.array([g["smax"], g["smax_no_clip"]])
    Wq2, Wk2, gamma, mask = oracle.qk_clip(Wq, Wk, smax, g["tau"], g["alpha"], H, dh)
    assert gamma[0] == pytest.approx(g["gamma"], abs=1e-15) and gamma[1] == 1.0
    assert list(mask) == [1, 0]
    assert np.allclose(Wq2[:dh], g["side_scale"] * Wq[:dh], rtol=1e-15, atol=0)
    assert np.allclose(Wk2[:dh], g["side_scale"] * Wk[:dh], rtol=1e-15, atol=0)
    assert np.array_equal(Wq2[dh:], Wq[dh:]) and np.array_equal(Wk2[dh:], Wk[dh:])


def test_clip_threshold_edges_leave_weights_bitwise():
    Wq = np.arange(12.0).reshape(4, 3); Wk = -Wq
    for s in (100.0, 99.999, -500.0, 0.0):
        q2, k2, gamma, mask = oracle.qk_clip(Wq, Wk, np.array([s, s]), 100.0, 0.5, 2, 2)
        assert np.array_equal(q2, Wq) and np.array_equal(k2, Wk)
        assert mask.sum() == 0 and np.all(gamma == 1.0)


@pytest.mark.parametrize("alpha", [0.5, 0.3, 1.0])
def test_recomputed_smax_after_clip_equals_tau(alpha):
    rng = np.random.default_rng(15)
    B, S, D, H, dh = 2, 12, 16, 3, 4
    X = rng.standard_normal((B, S, D))
    Wq = rng.standard_normal((H * dh, D)) * np.array([4.0] * dh + [0.1] * dh + [5.0] * dh)[:, None]
    Wk = rng.standard_normal((H * dh, D)) * np.array([4.0] * dh + [0.1] * dh + [5.0] * dh)[:, None]
    tau = 5.0
    s0 = oracle.qk_max_logit(X, Wq, Wk, H, dh)
    q2, k2, gamma, mask = oracle.qk_clip(Wq, Wk, s0, tau, alpha, H, dh)
    s1 = oracle.qk_max_logit(X, q2, k2, H, dh)
    for h in range(H):
        if s0[h] > tau:
            assert s1[h] == pytest.approx(tau, rel=1e-12)
            assert s1[h] <= tau * (1 + 1e-6)
        else:
            assert s1[h] == s0[h]
    assert mask.sum() >= 1


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(16)
    x = rng.standard_normal(10000) * np.exp(rng.uniform(-20, 20, 10000))
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x), want)


# ------------------------------------------------ per-step coefficient tables
def test_ns_coefficient_schedule_equals_composed_scalar_maps():
    """With a per-iteration schedule, the odd-polynomial identity composes:
    NS(U diag(s) V^T) = U diag(phi_N o ... o phi_1 (s/||s||)) V^T."""
    rng = np.random.default_rng(21)
    r, c = 30, 52
    U, V = haar(rng, r, r), haar(rng, c, r)
    s = np.sort(rng.uniform(0.02, 2.0, r))[::-1]
    G = (U * s) @ V.T
    sched = [tuple(GOLD["classic_cubic"]["value"])] * 2 + [tuple(GOLD["simple_quintic"]["value"])] * 3 + [TUNED] * 2
    got = oracle.newton_schulz(G, len(sched), *TUNED, coeffs=sched)
    want = (U * oracle.phi_schedule(s / np.linalg.norm(s), sched)) @ V.T
    assert np.linalg.norm(got - want) <= 1e-12 * np.linalg.norm(want)
    # a schedule of one repeated triple is the plain iteration
    same = oracle.newton_schulz(G, 5, *TUNED, coeffs=[TUNED] * 5)
    assert np.array_equal(same, oracle.newton_schulz(G, 5, *TUNED))


def test_cubic_schedule_converges_to_polar_factor():
    """The classic cubic (1.5, -0.5, 0) converges to exactly U V^T (printed:
    converges to exactly 1); numpy's SVD gives the polar factor."""
    rng = np.random.default_rng(22)
    G = rng.standard_normal((20, 35)) + 2 * np.eye(20, 35)
    u, _, vt = np.linalg.svd(G, full_matrices=False)
    cubic = tuple(GOLD["classic_cubic"]["value"])
    O = oracle.newton_schulz(G, 60, *TUNED, coeffs=[cubic] * 60)
    assert np.linalg.norm(O - u @ vt) <= 1e-9 * np.linalg.norm(u @ vt)


# ------------------------------------------------------------ MLA QK-Clip
def _mla_setup(seed=23, B=2, S=10, D=12, H=3, dc=4, dr=2):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((B, S, D))
    w = {"W_qC": rng.standard_normal((H * dc, D)), "W_kC": rng.standard_normal((H * dc, D)),
         "W_qR": rng.standard_normal((H * dr, D)), "W_kR": rng.standard_normal((dr, D))}
    return X, w, H, dc, dr


def test_mla_clip_worked_example():
    g = GOLD["mla_clip_example"]
    X, w, H, dc, dr = _mla_setup()
    smax = np.array([g["smax"], 50.0, 80.0])
    out, gamma, mask = oracle.qk_clip_slices(w, oracle.mla_slices(H, dc, dr), smax, g["tau"])
    assert gamma[0] == pytest.approx(g["gamma"], abs=1e-15) and list(mask) == [1, 0, 0]
    assert np.allclose(out["W_qC"][:dc], g["content_scale"] * w["W_qC"][:dc], rtol=1e-15, atol=0)
    assert np.allclose(out["W_kC"][:dc], g["content_scale"] * w["W_kC"][:dc], rtol=1e-15, atol=0)
    assert np.allclose(out["W_qR"][:dr], g["rotary_query_scale"] * w["W_qR"][:dr], rtol=1e-15, atol=0)
    assert np.array_equal(out["W_kR"], w["W_kR"])          # shared rotary key untouched
    for k in ("W_qC", "W_kC"):
        assert np.array_equal(out[k][dc:], w[k][dc:])      # other heads untouched
    assert np.array_equal(out["W_qR"][dr:], w["W_qR"][dr:])


def test_mla_recomputed_max_logit_equals_tau():
    """Both parts of the MLA score (content and rotary) scale by gamma, so a
    clipped head comes back to exactly tau; unclipped heads are unchanged."""
    X, w, H, dc, dr = _mla_setup(seed=24)
    w["W_qC"][:4] *= 6.0
    w["W_kC"][:4] *= 6.0
    w["W_qR"][:2] *= 20.0
    s0 = oracle.mla_max_logit(X, w, H, dc, dr)
    tau = float(np.sort(s0)[-1]) / 3
    out, gamma, mask = oracle.qk_clip_slices(w, oracle.mla_slices(H, dc, dr), s0, tau)
    s1 = oracle.mla_max_logit(X, out, H, dc, dr)
    assert mask.sum() >= 1
    for h in range(H):
        if mask[h]:
            assert s1[h] == pytest.approx(tau, rel=1e-12)
        else:
            assert s1[h] == pytest.approx(s0[h], rel=1e-14)


def test_mha_as_a_slice_map_equals_qk_clip():
    rng = np.random.default_rng(25)
    H, dh, D = 4, 3, 5
    Wq, Wk = rng.standard_normal((H * dh, D)), rng.standard_normal((H * dh, D))
    smax = np.array([300.0, 90.0, 101.0, -4.0])
    alpha = 0.3
    q2, k2, g1, m1 = oracle.qk_clip(Wq, Wk, smax, 100.0, alpha, H, dh)
    sl = [s for h in range(H) for s in (("q", h, h * dh, (h + 1) * dh, alpha), ("k", h, h * dh, (h + 1) * dh, 1 - alpha))]
    out, g2, m2 = oracle.qk_clip_slices({"q": Wq, "k": Wk}, sl, smax, 100.0)
    assert np.array_equal(out["q"], q2) and np.array_equal(out["k"], k2)
    assert np.array_equal(g1, g2) and np.array_equal(m1, m2)


def test_mla_max_logit_bruteforce_tiny():
    """The content + rotary split, with the rotary key shared by all heads,
    equals an explicit loop over every pair and feature on a tiny case."""
    X, w, H, dc, dr = _mla_setup(seed=26, B=1, S=5, D=4, H=2, dc=3, dr=2)
    got = oracle.mla_max_logit(X, w, H, dc, dr)
    want = np.full(H, -np.inf)
    for h in range(H):
        for i in range(5):
            for j in range(i + 1):
                s = 0.0
                for e in range(dc):
                    r = h * dc + e
                    s += (X[0, i] @ w["W_qC"][r]) * (X[0, j] @ w["W_kC"][r])
                for e in range(dr):
                    s += (X[0, i] @ w["W_qR"][h * dr + e]) * (X[0, j] @ w["W_kR"][e])
                want[h] = max(want[h], s / np.sqrt(dc + dr))
    assert np.allclose(got, want, rtol=1e-12)


def test_mla_with_zero_rotary_part_is_mha():
    """With the rotary weights zero, the MLA statistic is the MHA one over the
    content projections, rescaled from 1/sqrt(dc) to 1/sqrt(dc + dr)."""
    X, w, H, dc, dr = _mla_setup(seed=27)
    w["W_qR"][:] = 0.0
    w["W_kR"][:] = 0.0
    got = oracle.mla_max_logit(X, w, H, dc, dr)
    mha = oracle.qk_max_logit(X, w["W_qC"], w["W_kC"], H, dc)
    assert np.allclose(got, mha * np.sqrt(dc) / np.sqrt(dc + dr), rtol=1e-12)


# ------------------------------------------------------------ NorMuon
def _nm_hp(**kw):
    h = dict(wl.HPARAMS)
    h.update(beta2=0.95, eps_v=1e-8)
    h.update(kw)
    return h


def test_normuon_keeps_the_frobenius_norm_and_equalises_rows():
    """The two facts the page states: the update is rescaled to the Frobenius
    norm it had going in, and (with a fresh state) every row then carries the
    same share of it."""
    rng = np.random.default_rng(40)
    r, c = 24, 40
    W, G, M = rng.normal(0, 0.02, (r, c)), rng.normal(0, 1, (r, c)) * np.exp(rng.normal(0, 1, (r, 1))), np.zeros((r, c))
    h = _nm_hp(beta2=0.0, eps_v=0.0)
    _, _, upd_mu, _ = oracle.muon_step(W, G, M, **{k: v for k, v in h.items() if k not in ("beta2", "eps_v")})
    _, _, upd, v = oracle.normuon_step(W, G, M, np.zeros(r), **h)
    assert np.linalg.norm(upd) == pytest.approx(np.linalg.norm(upd_mu), rel=1e-12)
    rn = np.linalg.norm(upd, axis=1)
    assert np.allclose(rn, rn[0], rtol=1e-12)
    # the Muon update itself does not have equal rows here (the row scaling of G survives)
    rm = np.linalg.norm(upd_mu, axis=1)
    assert rm.max() / rm.min() > 1.01
    # the state holds the row mean squares of the NS output
    O = upd_mu / (h["rms_scale"] * np.sqrt(max(r, c)))
    assert np.allclose(v, np.mean(O * O, axis=1), rtol=1e-12)


def test_normuon_reduces_to_muon_when_rows_are_already_equal():
    """An exactly orthogonal square NS output (simple quintic run to
    convergence) has unit rows, so the row division is uniform and NorMuon is
    Muon; likewise with a large uniform state, whatever the rows."""
    rng = np.random.default_rng(41)
    n = 32
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    G = Q @ np.diag(np.linspace(1.0, 0.5, n)) @ np.linalg.qr(rng.standard_normal((n, n)))[0].T
    W, M = rng.normal(0, 0.02, (n, n)), np.zeros((n, n))
    simple = [(2.0, -1.5, 0.5)] * 40
    base = {k: v for k, v in _nm_hp().items() if k not in ("beta2", "eps_v")}
    base.update(ns_steps=40, coeffs=simple)
    W_mu, _, _, _ = oracle.muon_step(W, G, M, **base)
    W_nm, _, _, _ = oracle.normuon_step(W, G, M, np.zeros(n), beta2=0.95, eps_v=1e-8, **base)
    assert np.allclose(W_nm, W_mu, rtol=0, atol=1e-12)
    # any shape, large uniform prior state: v ~ beta2 * 1e6 on every row
    W, G, M = rng.normal(0, 0.02, (20, 36)), rng.normal(0, 1, (20, 36)), np.zeros((20, 36))
    base = {k: v for k, v in _nm_hp().items() if k not in ("beta2", "eps_v")}
    W_mu, _, _, _ = oracle.muon_step(W, G, M, **base)
    W_nm, _, _, _ = oracle.normuon_step(W, G, M, np.full(20, 1e6), beta2=0.95, eps_v=0.0, **base)
    assert np.allclose(W_nm, W_mu, rtol=0, atol=1e-9)


def test_normuon_fresh_state_is_independent_of_beta2():
    """With v0 = 0 the first state is (1 - beta2) times the row mean squares,
    a common factor that the Frobenius rescale removes."""
    rng = np.random.default_rng(42)
    W, G, M = rng.normal(0, 0.02, (30, 18)), rng.normal(0, 1, (30, 18)), rng.normal(0, 0.1, (30, 18))
    outs = [oracle.normuon_step(W, G, M, np.zeros(30), **_nm_hp(beta2=b2, eps_v=0.0)) for b2 in (0.0, 0.5, 0.95)]
    for o in outs[1:]:
        assert np.allclose(o[0], outs[0][0], rtol=0, atol=1e-13)
        assert np.allclose(o[2], outs[0][2], rtol=1e-10, atol=1e-13)


def test_normuon_worked_example_by_hand():
    """A 2 x 2 example worked out by hand, with a prior state.  O = [[3, -3],
    [1, 1]] has row mean squares (9, 1).  From v0 = (1, 4) with beta2 = 3/4:
    v1 = 3/4 (1, 4) + 1/4 (9, 1) = (3, 13/4).  Dividing the rows by sqrt(v1)
    gives (sqrt3, -sqrt3) and (1, 1)/sqrt(13/4), of squared norm 6 + 8/13 =
    86/13; ||O||_F^2 = 20, so both rows are then scaled by sqrt(20 * 13/86) =
    sqrt(130/43): O_hat = [[r0, -r0], [r1, r1]] with r0 = sqrt(390/43) and
    r1 = sqrt(40/43).  The weights swapped (1/4 on the state, 3/4 on the new
    mean square) would give v1 = (7, 7/4) instead."""
    O = np.array([[3.0, -3.0], [1.0, 1.0]])
    O_hat, v1 = oracle.normuon_rows(O, np.array([1.0, 4.0]), beta2=0.75, eps_v=0.0)
    assert np.allclose(v1, [3.0, 3.25], rtol=0, atol=1e-15)
    r0, r1 = np.sqrt(390.0 / 43.0), np.sqrt(40.0 / 43.0)
    assert np.allclose(O_hat, [[r0, -r0], [r1, r1]], rtol=1e-14, atol=0)


def test_normuon_second_moment_is_an_exponential_average():
    """Fed the same rows k times, an exponential average with factor beta2
    closes to the geometric series v_k = q + beta2^k (v0 - q), q being the
    row's mean square (here each row has entries of one magnitude c_i, so
    q = c_i^2 exactly).  A row whose prior state is far above q is therefore
    damped more, step after step, the larger beta2 is."""
    rng = np.random.default_rng(43)
    r, c = 6, 10
    mag = rng.uniform(0.5, 2.0, r)
    O = mag[:, None] * rng.choice([-1.0, 1.0], (r, c))
    v0 = rng.uniform(0.0, 20.0, r)
    for beta2 in (0.3, 0.9):
        v = v0.copy()
        for k in range(1, 6):
            _, v = oracle.normuon_rows(O, v, beta2=beta2, eps_v=1e-8)
            want = mag ** 2 + beta2 ** k * (v0 - mag ** 2)
            assert np.allclose(v, want, rtol=1e-13, atol=0), (beta2, k)
    # one step from a large prior state on row 0 only: row 0's share of the
    # (norm-preserving) update falls as beta2 grows
    v_big = np.full(r, 1.0)
    v_big[0] = 1e4
    share = []
    for beta2 in (0.1, 0.5, 0.9):
        O_hat, _ = oracle.normuon_rows(O, v_big, beta2=beta2, eps_v=0.0)
        share.append(np.linalg.norm(O_hat[0]) / np.linalg.norm(O_hat))
    assert share[0] > share[1] > share[2]


# ------------------------------------------------------------ Polar Express
def test_polar_express_ten_steps_printed_value():
    g = GOLD["polar_express_10"]
    sched = oracle.polar_express_schedule(g["steps"])
    assert len(sched) == 10
    assert float(oracle.phi_schedule(g["x0"], sched)) == pytest.approx(g["printed"], abs=g["tol"])
    # the five-step tuned quintic stays far below (the printed 0.05 of the same bullet)
    tuned = GOLD["tuned_coefficients"]["value"]
    assert float(oracle.phi_iter(g["x0"], 5, *tuned)) < 0.06


def test_minimax_quintic_is_optimal_against_a_linear_program():
    """The Remez result equioscillates at four points, and no odd quintic does
    better on a fine grid (an LP over (a, b, c, E), solved independently)."""
    from scipy.optimize import linprog
    for lo, hi in ((1e-3, 1.0), (0.3, 1.7), (0.05, 1.0)):
        (a, b, c), E = oracle.minimax_odd_quintic(lo, hi)
        x = np.linspace(lo, hi, 20001)
        err = 1.0 - (a * x + b * x ** 3 + c * x ** 5)
        assert np.max(np.abs(err)) == pytest.approx(E, rel=1e-6)
        # sign changes of the error at its extrema: at least 3 (4 alternation points)
        ext = np.r_[0, np.nonzero(np.diff(np.sign(np.diff(err))))[0] + 1, len(x) - 1]
        assert np.sum(np.diff(np.sign(err[ext])) != 0) >= 3
        # LP: minimise E s.t. |1 - (a x + b x^3 + c x^5)| <= E on the grid
        xg = np.linspace(lo, hi, 4001)
        V = np.stack([xg, xg ** 3, xg ** 5], axis=1)
        A_ub = np.block([[V, -np.ones((len(xg), 1))], [-V, -np.ones((len(xg), 1))]])
        b_ub = np.r_[np.ones(len(xg)), -np.ones(len(xg))]
        lp = linprog(c=[0, 0, 0, 1], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 4, method="highs")
        assert lp.status == 0
        assert lp.fun == pytest.approx(E, rel=1e-4)
        assert E <= lp.fun * (1 + 1e-4)


def test_minimax_limit_polynomial_on_a_shrinking_interval():
    """On [1 - d, 1 + d] the minimax quintic tends to the odd quintic with
    p(1) = 1 and p'(1) = p''(1) = 0, which the schedule uses once the
    interval is too narrow to resolve."""
    (a, b, c), E = oracle.minimax_odd_quintic(1 - 1e-3, 1 + 1e-3)
    assert (a, b, c) == pytest.approx((15 / 8, -10 / 8, 3 / 8), abs=1e-4)
    assert oracle.phi(1.0, 15 / 8, -10 / 8, 3 / 8) == pytest.approx(1.0, abs=1e-15)
    assert 15 / 8 - 3 * 10 / 8 + 5 * 3 / 8 == pytest.approx(0.0, abs=1e-15)     # p'(1)
    assert -6 * 10 / 8 + 20 * 3 / 8 == pytest.approx(0.0, abs=1e-15)            # p''(1)
